/*
 * mla_decode.h -- C ABI of the B200 (sm_100a) library for DeepSeek-style
 * Multi-head Latent Attention (MLA) decode over a paged latent KV cache,
 * computed through matrix absorption.
 *
 * The method ("MLA operator design" page, bhfrc.com/news/60867, §1 and §4;
 * "MHA2MLA" page, lpnh.cn/news/2494972, §2.1): per token and layer the cache
 * keeps a d_c-wide latent c_KV plus a d_R-wide decoupled-RoPE key k_R. A decode
 * step with query q = [q_c (d_n per head) | q_r (d_R per head)] computes, per
 * head h,
 *     out_h = softmax(scale * (q_c W_UK[h] c_KV^T + q_r k_R^T)) c_KV W_UV[h]
 * in four calls:
 *     mla_absorb_q        Q = [q_c W_UK[h] | q_r]                (fold into latent space)
 *     mla_decode_splitkv  per partition of the cache: o = softmax(Q [c_KV|k_R]^T) c_KV, lse
 *     mla_combine         log-sum-exp merge of the partitions -> o_lat
 *     mla_absorb_out      out = o_lat W_UV[h]                    (up-project once)
 * so the per-head K and V are never materialised.
 *
 * Conventions for every call:
 *   - All pointers are DEVICE pointers unless a parameter says "host". The
 *     caller owns every buffer; the library allocates no device memory.
 *   - bf16 means IEEE bfloat16 stored as 16-bit words; fp32 is float.
 *   - Tensors are dense row-major unless a stride is given. Shapes are written
 *     outermost first, e.g. [T, H, d] has d contiguous.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and never synchronise, except mla_get_device_error.
 *   - Argument errors are detected on the host before anything is launched and
 *     returned as MLA_ERR_INVALID_ARG / MLA_ERR_UNSUPPORTED; nothing is written
 *     in that case. Data-dependent errors found by the kernels (a page id
 *     outside the pool, a sequence length beyond its table row or below n_q, a
 *     bounded wait that ran out) are recorded in a device error word and read
 *     back with mla_get_device_error; the affected outputs are then undefined
 *     but every kernel still terminates.
 *   - Results are deterministic: repeated calls with the same inputs and the
 *     same num_parts give bitwise-identical outputs, independent of which
 *     physical pages hold the tokens.
 *   - Kernels are launched with programmatic dependent launch: each may start
 *     while the kernel ahead of it on the stream is still running, and waits
 *     for that kernel to finish before it reads that kernel's outputs. The
 *     decode calls read seq_lens and block_table before that wait, the
 *     combine calls seq_lens; the other calls read only their weights before
 *     it. The kernels of this library never write those inputs, so a stream
 *     that produces them with copies, with this library's calls or with
 *     kernels that do not trigger their dependents early is always safe; a
 *     custom kernel that triggers early (griddepcontrol.launch_dependents)
 *     must not write a call's seq_lens or block_table when it runs directly
 *     before that call.
 */
#ifndef MLA_DECODE_H
#define MLA_DECODE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MLA_OK = 0,
    MLA_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, bad size, inconsistent dims */
    MLA_ERR_UNSUPPORTED = 2,   /* dims outside the compiled specialisations, no sm_100 device */
    MLA_ERR_CUDA = 3,          /* a CUDA runtime call failed */
    MLA_ERR_DEVICE_BOUNDS = 4, /* (device word) bad page id or sequence length */
    MLA_ERR_TIMEOUT = 5        /* (device word) a bounded wait inside a kernel ran out */
} mla_status;

/* Problem dimensions. Supported specialisations:
 *   d_latent 512, d_rope 64   (DeepSeek-V2/V3: "MLA operator design" §3 constants)
 *   d_latent  64, d_rope  8   (retrofitted MLA: "MHA2MLA" §3.2 configuration)
 * with page_size 64, d_nope <= 128 and a multiple of 8, d_v <= 256 and a
 * multiple of 8, and n_q * num_heads <= 128 query rows per sequence. */
typedef struct {
    int32_t num_heads;     /* H */
    int32_t n_q;           /* query tokens per sequence in this step (1, or 2 for a causal pair) */
    int32_t d_nope;        /* d_n: per-head non-RoPE query width (128 or 120) */
    int32_t d_latent;      /* d_c: latent width of c_KV */
    int32_t d_rope;        /* d_R: width of the decoupled RoPE key k_R */
    int32_t d_v;           /* per-head value width (128) */
    int32_t page_size;     /* tokens per cache page; must be 64 ("MLA operator design" §3) */
    float softmax_scale;   /* <= 0 selects 1/sqrt(d_nope + d_rope) ("MLA operator design" §4) */
} mla_dims;

/* One page pool: element (page p, token j, channel c) is at
 * base[p * page_stride + j * token_stride + c] (strides in elements).
 * base must be 16-byte aligned and both strides multiples of 8 elements
 * (16 bytes), as the tensor-memory-access engine requires. The c_KV and k_R
 * pools may be separate tensors or two views of one interleaved
 * [pages, 64, d_c + d_R] tensor. */
typedef struct {
    const void *base;
    int64_t page_stride;
    int64_t token_stride;
} mla_pool;

/*
 * Absorb-in ("MLA operator design" §4, path B: q_abs = q_c . w_uk per head).
 *   q_out[t, h, 0:d_c]       = bf16( sum_d q_c[t, h, d] * w_uk[h, d, :] )   (fp32 accumulation)
 *   q_out[t, h, d_c:d_c+d_R] = q_r[t, h, :]                                 (bit copy)
 * q_c   [T, H, d_nope] bf16      q_r  [T, H, d_rope] bf16
 * w_uk  [H, d_nope, d_latent] bf16 (the page's w_uk[nh, dhc, dc] layout)
 * q_out [T, H, d_latent + d_rope] bf16; T = num_tokens >= 0 (0 is a no-op).
 * All pointers 16-byte aligned.
 */
mla_status mla_absorb_q(const mla_dims *dims, const void *q_c, const void *q_r, const void *w_uk,
                        void *q_out, int32_t num_tokens, void *stream);

/* Number of cache partitions mla_decode_splitkv should use for a batch whose
 * sequences hold total_tiles tiles in all (sum of ceil(L_b / tile), tile = 64
 * tokens for d_latent 512, 128 for d_latent 64), on a device with num_sms
 * multiprocessors: min(ceil(total_tiles / 8), num_sms / 2) for d_latent 512
 * (at most one per CTA pair), min(total_tiles, num_sms) for d_latent 64.
 * Host-only arithmetic; returns >= 1. */
int32_t mla_decode_num_parts(const mla_dims *dims, int64_t total_tiles, int32_t num_sms);

/* Bytes of device workspace mla_decode_splitkv / mla_combine need for `batch`
 * sequences and `num_parts` partitions. Layout (R = n_q * num_heads,
 * S = batch + num_parts slots):
 *   offset 0:                 o_part [S, R, d_latent] fp32 (normalised partial outputs)
 *   offset align256(S*R*d_c*4): lse_part [S, R] fp32 (natural-log log-sum-exp of
 *                             the scaled scores of each partial; -inf if empty)
 * Returns 0 for invalid dims. */
size_t mla_decode_workspace_bytes(const mla_dims *dims, int32_t batch, int32_t num_parts);

/* The same two sizing helpers in split-KV terms (a split is one partition),
 * sized from the batch and its longest sequence instead of the tile total:
 *   mla_default_num_splits(dims, batch, max_seq_len, num_sms)
 *       = mla_decode_num_parts(dims, batch * ceil(max_seq_len / tile), num_sms)
 *     with tile = 64 tokens (d_latent 512) or 128 (d_latent 64), i.e. the
 *     partition count for `batch` sequences of at most max_seq_len tokens;
 *     returns >= 1 (1 for invalid arguments).
 *   mla_decode_workspace_size(dims, batch, num_splits)
 *       = mla_decode_workspace_bytes(dims, batch, num_splits).
 * The partials of every split live inside the workspace at the layout given
 * above, so mla_decode_splitkv and mla_combine take the workspace instead of
 * separate partial-output pointers. */
int32_t mla_default_num_splits(const mla_dims *dims, int32_t batch, int32_t max_seq_len,
                               int32_t num_sms);
size_t mla_decode_workspace_size(const mla_dims *dims, int32_t batch, int32_t num_splits);

/*
 * Split-KV decode in latent space (the absorbed score and value steps).
 * The tiles of all sequences (N tiles of 64 tokens for d_latent 512, of 128
 * tokens for d_latent 64) are laid end to end with W virtual tiles between
 * consecutive non-empty sequences (W = 8 for 64-token tiles, 3 for 128-token
 * tiles: the cost of switching to another sequence inside a range, a Q load
 * and a partial-result write). The C = N + W (sequences - 1) positions are cut
 * into P = min(num_parts, N) contiguous ranges, range p holding positions
 * [floor(p C / P), floor((p+1) C / P)), and each range's real tiles are
 * processed by one CTA pair (d_latent 512) or one CTA (d_latent 64); a range
 * that lies inside a gap has none. For every (sequence, range) overlap it
 * writes one slot of the workspace, slots numbered sequence-major:
 *   s[r, t]  = scale * (Q[b, r, 0:d_c] . c_KV[t] + Q[b, r, d_c:] . k_R[t])
 *   o[r, :]  = sum_t softmax(s[r, :])_t c_KV[t]       over the range's visible tokens
 *   lse[r]   = log sum_t exp(s[r, t])
 * Row r = i * H + h of sequence b is query i (0 <= i < n_q) of head h; it sees
 * tokens t <= seq_lens[b] - n_q + i (seq_lens counts the tokens already in the
 * cache, the n_q current ones included).
 * Token t of sequence b is read from page block_table[b * max_pages_per_seq + t / 64],
 * row t % 64 ("MLA operator design" §3 page table); entries past
 * ceil(seq_lens[b] / 64) are never read.
 *
 * q           [batch, n_q * H, d_latent + d_rope] bf16 (the q_out of mla_absorb_q)
 * ckv, kr     page pools (host structs describing device memory), num_pages pages each
 * block_table [batch, max_pages_per_seq] int32
 * seq_lens    [batch] int32, n_q <= seq_lens[b] <= max_pages_per_seq * 64
 * workspace   >= mla_decode_workspace_bytes(dims, batch, num_parts) bytes, 256-byte aligned
 * batch = 0 is a no-op.
 */
mla_status mla_decode_splitkv(const mla_dims *dims, const void *q, const mla_pool *ckv,
                              const mla_pool *kr, int32_t num_pages, const int32_t *block_table,
                              int32_t max_pages_per_seq, const int32_t *seq_lens, int32_t batch,
                              int32_t num_parts, void *workspace, size_t workspace_bytes,
                              void *stream);

/*
 * Log-sum-exp merge of the partial results written by mla_decode_splitkv with
 * the same dims, seq_lens, batch and num_parts:
 *   L = log sum_s exp(lse_s),   o_lat[b, r, :] = bf16( sum_s exp(lse_s - L) o_s[r, :] )
 * A row with no visible token gives o_lat = 0 and lse = -inf.
 * o_lat   [batch, n_q * H, d_latent] bf16 (= [batch, n_q, H, d_latent])
 * lse_out [batch, n_q * H] fp32, may be NULL.
 */
mla_status mla_combine(const mla_dims *dims, const void *workspace, size_t workspace_bytes,
                       const int32_t *seq_lens, int32_t max_pages_per_seq, int32_t batch,
                       int32_t num_parts, void *o_lat, float *lse_out, void *stream);

/*
 * Absorb-in with the rotary embedding of the RoPE part fused in: as
 * mla_absorb_q, except that q_r arrives unrotated and
 *   q_out[t, h, d_latent + 2i]     = bf16(x0 cos(a) - x1 sin(a))
 *   q_out[t, h, d_latent + 2i + 1] = bf16(x0 sin(a) + x1 cos(a))
 * with (x0, x1) = q_r[t, h, 2i .. 2i + 1] and a = positions[t] *
 * rope_theta^(-2i / d_rope) ("MHA2MLA" §3.2, rope_theta 10000; the "MLA
 * operator design" page §3 computes RoPE in fp32: here the angle and its
 * reduction are fp64, the rotation fp32). The pairing of adjacent channels is
 * this library's reading of a convention the pages leave unstated.
 * positions [num_tokens] int32 device (the token's absolute position, e.g.
 * seq_len - n_q + i for query i of a sequence); a negative entry is treated as
 * 0 and sets MLA_ERR_DEVICE_BOUNDS in the device error word. rope_theta must
 * be finite and > 1 (MLA_ERR_INVALID_ARG otherwise). The latent part is
 * identical to mla_absorb_q's.
 */
mla_status mla_absorb_q_rope(const mla_dims *dims, const void *q_c, const void *q_r,
                             const void *w_uk, const int32_t *positions, float rope_theta,
                             void *q_out, int32_t num_tokens, void *stream);

/*
 * Absorb-out ("MHA2MLA" §2.1: v = c_kv W_uv, applied once to the latent result).
 *   out[t, h, :] = bf16( sum_c o_lat[t, h, c] * w_uv[h, c, :] )   (fp32 accumulation)
 * o_lat [T, H, d_latent] bf16, w_uv [H, d_latent, d_v] bf16, out [T, H, d_v] bf16.
 */
mla_status mla_absorb_out(const mla_dims *dims, const void *o_lat, const void *w_uv, void *out,
                          int32_t num_tokens, void *stream);

/*
 * Combine and absorb-out in one call (the merge of mla_combine followed by the
 * W_UV product of mla_absorb_out, "MHA2MLA" §2.1), without writing o_lat:
 *   L = logsumexp_s lse_s,  o_lat = sum_s exp(lse_s - L) o_s   (as mla_combine)
 *   out[t, h, :] = bf16( sum_c bf16(o_lat[t, h, c]) * w_uv[h, c, :] )
 * over the tokens t = b * n_q + i of the batch. Arguments as mla_combine, plus
 * w_uv [H, d_latent, d_v] bf16 and out [batch * n_q, H, d_v] bf16 (device,
 * caller-owned, 16-byte aligned); lse_out [batch * n_q, H] fp32 may be NULL.
 * The K sum may split d_latent into 128-channel parts reduced in a fixed
 * order, so the result can differ from mla_combine + mla_absorb_out in the
 * last bit of a bf16 output; repeated calls are bitwise identical.
 * Supported: d_v <= 128, d_latent 64, 128 or a multiple of 128 up to 1024,
 * num_parts < 160 (MLA_ERR_UNSUPPORTED otherwise); MLA_ERR_INVALID_ARG on null/misaligned
 * pointers or a workspace smaller than mla_decode_workspace_bytes.
 */
mla_status mla_combine_absorb_out(const mla_dims *dims, const void *workspace,
                                  size_t workspace_bytes, const int32_t *seq_lens,
                                  int32_t max_pages_per_seq, int32_t batch, int32_t num_parts,
                                  const void *w_uv, void *out, float *lse_out, void *stream);

/* Synchronises `stream`, returns in *code (host pointer) the first error a
 * kernel of this library recorded on the current device since the last call
 * (MLA_OK if none), and clears it. */
mla_status mla_get_device_error(int32_t *code, void *stream);

/* Static, human-readable name of a status code. */
const char *mla_status_string(int32_t status);

/*
 * Host-side partition plan, the same arithmetic the kernels use. For
 * seq_lens_host[batch] (host array) and num_parts, fills (host arrays, any may
 * be NULL):
 *   part_first[b]  first partition that covers sequence b (-1 if it has no tile)
 *   slot_count[b]  number of partial slots of sequence b
 *   slot_base[b]   index of its first slot in the workspace
 * and returns the total number of slots used (<= batch + num_parts), or -1 on
 * invalid arguments.
 */
int64_t mla_decode_plan(const mla_dims *dims, const int32_t *seq_lens_host,
                        int32_t max_pages_per_seq, int32_t batch, int32_t num_parts,
                        int32_t *part_first, int32_t *slot_count, int64_t *slot_base);

/*
 * Split-KV decode plus log-sum-exp combine (mla_decode_splitkv followed by
 * mla_combine) that allocates nothing and needs no workspace from the caller.
 * This entry point has no counterpart on the pages; it exists for callers that
 * cannot hand out device memory at call time -- for example a plugin's enqueue
 * routine inside an inference engine that owns the whole memory budget, or a
 * latency-critical path where a cudaMalloc (and the device synchronisation it
 * can imply) is not acceptable.
 * The partial results live in a fixed scratch array of MLA_NOALLOC_SCRATCH_BYTES
 * (32 MiB) that the library keeps in device memory on every GPU where it is
 * loaded, for the life of the process. Problems whose workspace
 * (mla_decode_workspace_bytes) exceeds it are rejected with
 * MLA_ERR_INVALID_ARG; nothing is launched then.
 * The first call on a device looks up that device's copy of the array
 * (cudaGetSymbolAddress), so make the first call on each device before any
 * stream capture. All calls share the one array and it keeps whatever the last
 * call left; every slot a call reads is written earlier by the same call, so
 * nothing needs clearing, but calls whose kernels overlap on the GPU (different
 * streams, no ordering between them) race on it and must be serialised by the
 * caller. Arguments and outputs are those of mla_decode_splitkv and mla_combine.
 */
#define MLA_NOALLOC_SCRATCH_BYTES (32u << 20)
mla_status mla_decode_latent_noalloc(const mla_dims *dims, const void *q, const mla_pool *ckv,
                                     const mla_pool *kr, int32_t num_pages,
                                     const int32_t *block_table, int32_t max_pages_per_seq,
                                     const int32_t *seq_lens, int32_t batch, int32_t num_parts,
                                     void *o_lat, float *lse_out, void *stream);

/*
 * Debug gather, the check on the page lookup of the decode calls: token t of
 * sequence b is row t % 64 of page block_table[b][t / 64] of the pool
 * ("MLA operator design" page §3, its 64-token pages). Uses the same TMA pool
 * descriptor construction and table lookup as mla_decode_splitkv and writes
 *   out[b, t, :] = pool[block_table[b][t / 64]][t % 64][0 : width]   (bit copy)
 * for t < seq_lens[b]; rows t >= seq_lens[b] of out are left untouched.
 * pool: base 16-byte aligned, strides in elements, multiples of 8, token
 * stride >= width. width: 8..512, a multiple of 8, and of 64 when above 64.
 * block_table [batch, max_pages_per_seq] int32, seq_lens [batch] int32 and
 * out [batch, max_len, width] bf16 are device pointers owned by the caller.
 * Returns MLA_ERR_INVALID_ARG on bad sizes or pointers (nothing launched);
 * a page id outside [0, num_pages) or seq_lens[b] outside [0, max_len] (or
 * beyond max_pages_per_seq pages) sets MLA_ERR_DEVICE_BOUNDS in the device
 * error word. Table entries past a sequence's last page are never read.
 */
mla_status mla_debug_gather(const mla_pool *pool, int32_t width, int32_t num_pages,
                            const int32_t *block_table, int32_t max_pages_per_seq,
                            const int32_t *seq_lens, int32_t batch, int32_t max_len, void *out,
                            void *stream);

/*
 * Test hook for the bounded waits: launches one block that waits on a barrier
 * nothing will complete, with a limit of timeout_ns nanoseconds, after which it
 * records MLA_ERR_TIMEOUT in the device error word and returns. Lets a test
 * check that a wait which runs out ends the kernel cleanly with a readable
 * status.
 */
mla_status mla_debug_wait_timeout(int64_t timeout_ns, void *stream);

/* ------------------------------------------------------------------------
 * Prefill through the decompress branch.
 *
 * The "MLA operator design" page (§3 constant kPrefillThresh, §6 threshold
 * sweep) routes a step by its query count M: M >= MLA_PREFILL_THRESHOLD takes
 * the decompress path (path A of §4: K_nope = c_KV W_UK[h]^T and
 * V = c_KV W_UV[h] per head, "MHA2MLA" page §2.1), below it the absorbed
 * decode path above. With many queries the per-head widths (d_n + d_R = 192,
 * d_v = 128) cost fewer FLOPs per (query, key, head) than the latent ones
 * (576, 512). Compiled specialisation: d_latent 512, d_rope 64, d_nope 128,
 * d_v 128, page_size 64 (MLA_ERR_UNSUPPORTED otherwise). dims->n_q is M.
 * The M queries of sequence b are its last M tokens: query i sits at position
 * seq_lens[b] - M + i and sees tokens t <= seq_lens[b] - M + i (causal).
 * ------------------------------------------------------------------------ */
#define MLA_PREFILL_THRESHOLD 256

/* Bytes of the decompressed-cache workspace for `batch` sequences of at most
 * max_pages_per_seq pages. Layout, with Lpad = max_pages_per_seq * 64 rounded
 * up to a multiple of 128 and half = align256(batch * H * Lpad * 128 * 2):
 *   offset 0:     K_nope [batch, H, Lpad, 128] bf16
 *   offset half:  V      [batch, H, Lpad, 128] bf16
 * Returns 0 for unsupported dims or bad sizes. */
size_t mla_prefill_workspace_bytes(const mla_dims *dims, int32_t batch, int32_t max_pages_per_seq);

/*
 * Decompression ("MHA2MLA" §2.1): for every sequence b, head h and token
 * t < round_up(seq_lens[b], 128),
 *   K_nope[b, h, t, d] = bf16( sum_c c_KV[t, c] W_UK[h, d, c] )
 *   V[b, h, t, e]      = bf16( sum_c c_KV[t, c] W_UV[h, c, e] )
 * with fp32 accumulation; rows t >= seq_lens[b] are written as zeros. Rows at
 * or past round_up(seq_lens[b], 128) are not written.
 * w_uk [H, 128, 512], w_uv [H, 512, 128] bf16 (16-byte aligned); the pool and
 * table as for mla_decode_splitkv; workspace 256-byte aligned, at least
 * mla_prefill_workspace_bytes. A page id outside [0, num_pages) or a length
 * outside [0, max_pages_per_seq * 64] sets MLA_ERR_DEVICE_BOUNDS.
 */
mla_status mla_decompress_kv(const mla_dims *dims, const mla_pool *ckv, int32_t num_pages,
                             const int32_t *block_table, int32_t max_pages_per_seq,
                             const int32_t *seq_lens, int32_t batch, const void *w_uk,
                             const void *w_uv, void *workspace, size_t workspace_bytes,
                             void *stream);

/*
 * Causal attention over the decompressed cache written by mla_decompress_kv
 * (same dims, table, lengths and workspace), for query i of sequence b and
 * head h:
 *   s[t]   = scale * (q_c[b, i, h, :] . K_nope[b, h, t, :] + q_r[b, i, h, :] . k_R[t, :])
 *   out[b, i, h, :] = bf16( sum_t softmax(s)_t V[b, h, t, :] ),  t <= seq_lens[b] - M + i
 *   lse[b, i, h]    = log sum_t exp(s[t])            (natural log; lse may be NULL)
 * q_c [batch, M, H, 128], q_r [batch, M, H, 64] bf16 (q_r already rotated, as
 * the cached k_R is); out [batch, M, H, 128] bf16; lse [batch, M, H] fp32.
 * scale = dims->softmax_scale, or 1/sqrt(d_nope + d_rope) when <= 0. A length
 * below M or beyond the table sets MLA_ERR_DEVICE_BOUNDS.
 */
mla_status mla_prefill_attention(const mla_dims *dims, const void *q_c, const void *q_r,
                                 const mla_pool *kr, int32_t num_pages, const int32_t *block_table,
                                 int32_t max_pages_per_seq, const int32_t *seq_lens, int32_t batch,
                                 const void *workspace, size_t workspace_bytes, void *out,
                                 float *lse, void *stream);

/* mla_decompress_kv followed by mla_prefill_attention on the same stream. */
mla_status mla_prefill(const mla_dims *dims, const void *q_c, const void *q_r, const mla_pool *ckv,
                       const mla_pool *kr, int32_t num_pages, const int32_t *block_table,
                       int32_t max_pages_per_seq, const int32_t *seq_lens, int32_t batch,
                       const void *w_uk, const void *w_uv, void *workspace,
                       size_t workspace_bytes, void *out, float *lse, void *stream);

/*
 * Cache write ("MLA operator design" page §3: paged latent cache, page_size
 * 64, RoPE computed in fp32; "MHA2MLA" page §3.2: rope_theta): for each new
 * token t with sequence b = seq_ids[t] and absolute position p = positions[t],
 *   c_KV pool [block_table[b][p / 64]][p % 64][:] = ckv_new[t, :]      (bit copy)
 *   k_R  pool [block_table[b][p / 64]][p % 64][:] = RoPE(kr_new[t, :], p)
 * RoPE turns channel pair (2i, 2i + 1) by p * rope_theta^(-2i / d_rope), angle
 * and its reduction in fp64, rotation fp32, result bf16 -- the same arithmetic
 * as mla_absorb_q_rope's q_r, so cached keys and queries rotate alike. With
 * rope_theta <= 0, k_R is copied unrotated. ckv_new [T, d_latent] bf16
 * (16-byte aligned), kr_new [T, d_rope] bf16 (unrotated), seq_ids / positions
 * [T] int32; pools and table as for mla_decode_splitkv (the c_KV pool needs a
 * 16-byte aligned base and strides that are multiples of 8 elements). Every
 * other slot of the pools is left untouched; two tokens aimed at the same slot
 * leave one of them there. A sequence id outside [0, batch), a position outside
 * [0, max_pages_per_seq * 64) or a page id outside [0, num_pages) skips that
 * token and sets MLA_ERR_DEVICE_BOUNDS.
 */
mla_status mla_append_kv(const mla_dims *dims, const void *ckv_new, const void *kr_new,
                         const int32_t *seq_ids, const int32_t *positions, int32_t num_tokens,
                         float rope_theta, const mla_pool *ckv, const mla_pool *kr,
                         int32_t num_pages, const int32_t *block_table, int32_t max_pages_per_seq,
                         int32_t batch, void *stream);

/* ------------------------------------------------------------------------
 * Low-precision latent cache. The "MLA operator design" page (introduction
 * and §5) gathers a quantised latent cache with 16-byte vector loads but does
 * not give the format; this library stores c_KV as fp8 E4M3 codes (the OCP
 * 8-bit floating-point format: bias 7, 3 mantissa bits, largest finite 448)
 * with one fp32 scale per cached token, and keeps k_R in bf16:
 *   codes pool [pages, 64, d_latent] uint8 (mla_pool strides in bytes, base
 *   and strides multiples of 16), scales [pages, 64] fp32 (dense).
 * Quantisation of a row x (IEEE fp32 throughout):
 *   amax = max |x|;  inv = 448 / amax;  code = E4M3_rn_satfinite(x * inv);
 *   scale = amax / 448          (an all-zero row: codes 0, scale 1)
 * Dequantisation: bf16_rn( fp32_rn( value(code) * scale ) ).
 * ------------------------------------------------------------------------ */

/* mla_append_kv writing the E4M3 cache: c_KV rows are quantised as above into
 * the codes pool and their scale into scales[page * 64 + slot]; k_R as in
 * mla_append_kv. d_latent must be a multiple of 16. */
mla_status mla_append_kv_fp8(const mla_dims *dims, const void *ckv_new, const void *kr_new,
                             const int32_t *seq_ids, const int32_t *positions, int32_t num_tokens,
                             float rope_theta, const mla_pool *ckv8, float *scales,
                             const mla_pool *kr, int32_t num_pages, const int32_t *block_table,
                             int32_t max_pages_per_seq, int32_t batch, void *stream);

/* Dequantising gather: out[b, t, :] = dequant(codes of token t of sequence b)
 * for t < seq_lens[b], bf16 [batch, max_len, width]; other rows untouched.
 * width: a multiple of 16, at most 4096. Bad page ids or lengths set
 * MLA_ERR_DEVICE_BOUNDS. */
mla_status mla_gather_dequant_fp8(const mla_pool *ckv8, const float *scales, int32_t width,
                                  int32_t num_pages, const int32_t *block_table,
                                  int32_t max_pages_per_seq, const int32_t *seq_lens,
                                  int32_t batch, int32_t max_len, void *out, void *stream);

/* mla_decompress_kv reading the E4M3 cache: the c_KV tile is dequantised as
 * above before the products, so the result equals mla_decompress_kv on the
 * dequantised bf16 cache. Use mla_prefill_attention afterwards as usual. */
mla_status mla_decompress_kv_fp8(const mla_dims *dims, const mla_pool *ckv8, const float *scales,
                                 int32_t num_pages, const int32_t *block_table,
                                 int32_t max_pages_per_seq, const int32_t *seq_lens, int32_t batch,
                                 const void *w_uk, const void *w_uv, void *workspace,
                                 size_t workspace_bytes, void *stream);

/* mla_decode_splitkv reading the E4M3 cache (the quantised latent-cache gather
 * that the "MLA operator design" page places on the decode side, introduction
 * and §5): c_KV comes from the codes pool and its per-token scales, k_R from
 * the bf16 pool. Each c_KV element is dequantised as above before it enters
 * either product, so the result is mla_decode_splitkv's on the dequantised
 * bf16 cache: HBM traffic per cached token is 512 code bytes + a 4-byte scale
 * + 128 bytes of k_R (644) instead of 1152. Elements past a sequence's end in
 * its last page never reach a product, whatever their codes or scale.
 * d_latent 512 / d_rope 64 only (else MLA_ERR_UNSUPPORTED); the workspace,
 * partition plan and the other arguments are those of mla_decode_splitkv, and
 * mla_combine reads the workspace unchanged.
 * ckv8    codes pool [pages, 64, >= 512] uint8 (strides in bytes, base and
 *         strides multiples of 16)
 * scales  [num_pages, 64] fp32, dense, 16-byte aligned base
 */
mla_status mla_decode_splitkv_fp8(const mla_dims *dims, const void *q, const mla_pool *ckv8,
                                  const float *scales, const mla_pool *kr, int32_t num_pages,
                                  const int32_t *block_table, int32_t max_pages_per_seq,
                                  const int32_t *seq_lens, int32_t batch, int32_t num_parts,
                                  void *workspace, size_t workspace_bytes, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* MLA_DECODE_H */
