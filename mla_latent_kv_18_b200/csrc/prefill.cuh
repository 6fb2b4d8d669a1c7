// Prefill through the decompress branch on sm_100a tensor cores.
//
// A step with M query tokens per sequence at or above the prefill threshold
// (the "MLA operator design" page §3 and §6: 256) re-expands the latent cache
// per head instead of folding the queries into it, because with many queries
// the per-head width (d_n + d_R = 192 for scores, d_v = 128 for values) costs
// fewer FLOPs than the latent width (576 and 512). Two kernels:
//
//  * decompress_kernel: K_nope[b,h,t,:] = c_KV[t] W_UK[h]^T and
//    V[b,h,t,:] = c_KV[t] W_UV[h] ("MHA2MLA" page §2.1). A CTA pair covers two
//    128-token tiles: each CTA keeps its tile of c_KV (128 tokens x 512
//    channels, two pages) in shared memory and streams its half of W_UK[h] /
//    W_UV[h] in 64-channel chunks through a TMA ring for each head of its
//    group; the leader accumulates both products with 2-SM tcgen05 MMAs
//    (M = 256) into double-buffered tensor-memory tiles, so that the epilogue
//    of one head overlaps the MMAs of the next.
//  * prefill_attn_kernel: causal attention of 128 queries of one (sequence,
//    head) against the decompressed keys [K_nope | k_R] and values V: scores
//    in tensor memory (two buffers), fp32 online softmax in the exp2 domain by
//    four warps (one query row per thread), P written back to tensor memory as
//    bf16 and used as the A operand of the P.V MMA, so it never touches shared
//    memory.
//
// Every wait is bounded; data errors set the device error word.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "decode.cuh"
#include "small_kernels.cuh"

namespace mla {

// ===========================================================================
// decompress_kernel
// ===========================================================================
namespace dkv {
constexpr int TOK = 128;                         // tokens per CTA tile (two pages)
constexpr int DC = 512, DN = 128, DV = 128;
constexpr int CHUNKS = DC / 64;                  // 64-channel K chunks
constexpr uint32_t A_BYTES = TOK * DC * 2;       // 8 swizzled blocks [128 tok x 64 ch]
// per CTA of the pair, half of each W chunk: W_UK rows d = 64 r .. 64 r + 63 (K-major
// [64 d x 64 c]) and W_UV columns e = 64 r .. 64 r + 63 (one MN-major [64 c x 64 e] block)
constexpr uint32_t WK_BYTES = 64 * 128;
constexpr uint32_t WV_BYTES = 64 * 128;
constexpr uint32_t STAGE_BYTES = WK_BYTES + WV_BYTES;   // 16384
constexpr int STAGES = 6;
constexpr uint32_t OFF_A = 0;
constexpr uint32_t OFF_STAGE = A_BYTES;
constexpr uint32_t OFF_MISC = OFF_STAGE + STAGES * STAGE_BYTES;
constexpr uint32_t MISC_BYTES = 1024;
constexpr uint32_t SMEM_BYTES = OFF_MISC + MISC_BYTES;   // the base is 1 KB aligned (checked)
constexpr uint32_t TMEM_COLS = 512;              // two buffers of [K_nope 128 | V 128]
// 2-SM MMAs: M = 256 (each CTA's 128 tokens), N = 128 split 64 / 64 between the CTAs
constexpr uint32_t IDESC_K = ptx::idesc_bf16(256, DN, 0, 0);
constexpr uint32_t IDESC_V = ptx::idesc_bf16(256, DV, 0, 1);
constexpr int THREADS = 192;                     // warp 0 TMA, warp 1 MMA (leader), warps 2..5 epilogue
static_assert(SMEM_BYTES <= 232448, "smem");
static_assert((OFF_STAGE % 1024) == 0 && (STAGE_BYTES % 1024) == 0, "align");

struct Misc {
    uint64_t a_full;                 // leader: both CTAs' c_KV tiles landed
    uint64_t w_full[STAGES];         // leader: both halves of a W chunk landed
    uint64_t w_empty[STAGES];        // each CTA: the chunk's MMAs are done
    uint64_t d_full[2];              // each CTA: a head's products are in tensor memory
    uint64_t d_free[2];              // leader: both CTAs' epilogues have read them
    uint64_t drain;
    uint32_t tmem_base;
    int32_t abort_flag;
};
static_assert(sizeof(Misc) <= MISC_BYTES, "misc");
}  // namespace dkv

struct DecompressArgs {
    const uint8_t *ckv8;         // E4M3 cache: pool base (kFp8 only)
    const float *scales;         // E4M3 cache: [pages, 64] per-token scales (kFp8 only)
    int64_t ckv8_page_stride, ckv8_token_stride;   // bytes
    const int32_t *block_table;  // [B, max_pages]
    const int32_t *seq_lens;     // [B]
    __nv_bfloat16 *k_nope;       // [B, H, Lpad, 128]
    __nv_bfloat16 *v;            // [B, H, Lpad, 128]
    int64_t timeout_ns;
    int32_t batch, heads, max_pages, num_pages, l_pad, pairs_per_seq, heads_per_cta;
};

// A CTA pair (cluster of two) covers tiles 2p and 2p + 1 of a sequence for a group
// of heads; the leader issues 2-SM MMAs with M = 256, each CTA supplying its own
// 128-token c_KV tile (A) and half of every W chunk (B), so each SM streams half
// the weight bytes of a one-CTA design for the same work. kFp8: the c_KV tiles
// come from the E4M3 cache; the epilogue warps dequantise them into the resident
// shared-memory tile before the first MMA (bf16(value(code) * scale)), so the rest
// is unchanged. map_ckv is unused then.
template <bool kFp8>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(dkv::THREADS, 1)
    decompress_kernel(const __grid_constant__ CUtensorMap map_ckv,
                      const __grid_constant__ CUtensorMap map_wuk,
                      const __grid_constant__ CUtensorMap map_wuv, const DecompressArgs args) {
    using namespace dkv;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t base = ptx::smem_u32(smem_raw);
    if (base & 1023u) {            // swizzled operands need a 1 KB aligned base; uniform over the pair
        if (threadIdx.x == 0) record_error(kErrUnsupported);
        return;
    }
    dkv::Misc *misc = reinterpret_cast<dkv::Misc *>(smem_raw + OFF_MISC);
    volatile int32_t *abort_flag = &misc->abort_flag;
    auto bar = [&](const uint64_t *b) { return ptx::smem_u32(b); };
    auto leader_bar = [&](const uint64_t *b) { return ptx::mapa(ptx::smem_u32(b), 0); };

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = ptx::cluster_ctarank();      // 0 = leader
    const int32_t pair = blockIdx.x >> 1;
    const int32_t b = pair / args.pairs_per_seq;
    const int32_t tb = 2 * (pair - b * args.pairs_per_seq) + static_cast<int32_t>(rank);
    const int32_t h0 = blockIdx.y * args.heads_per_cta;
    const int32_t nh = min(args.heads_per_cta, args.heads - h0);
    const int32_t L = args.seq_lens[b];
    // early exits are uniform over the pair (same sequence, same head group)
    if (L < 0 || static_cast<int64_t>(L) > static_cast<int64_t>(args.max_pages) * 64) {
        if (threadIdx.x == 0 && rank == 0 && tb == 0 && blockIdx.y == 0) record_error(kErrDeviceBounds);
        return;
    }
    if (TOK * (tb - static_cast<int32_t>(rank)) >= L || nh <= 0) return;   // the pair's first tile
    const int32_t rows_written = (L + TOK - 1) / TOK * TOK;   // rows >= L of the last tile are zeros
    const int32_t npages = (L + 63) / 64;

    if (threadIdx.x == 0) {
        ptx::mbar_init(bar(&misc->a_full), kFp8 ? 8 : 1);
        for (int i = 0; i < STAGES; ++i) {
            ptx::mbar_init(bar(&misc->w_full[i]), 1);
            ptx::mbar_init(bar(&misc->w_empty[i]), 1);
        }
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(bar(&misc->d_full[i]), 1);
            ptx::mbar_init(bar(&misc->d_free[i]), 8);
        }
        ptx::mbar_init(bar(&misc->drain), 1);
        misc->abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 1) {
        ptx::tmem_alloc<2>(bar(reinterpret_cast<uint64_t *>(&misc->tmem_base)), TMEM_COLS);
        ptx::tmem_relinquish<2>();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::cluster_sync();
    ptx::tc_fence_after();
    const uint32_t tmem = misc->tmem_base;
    const int total = nh * CHUNKS;                 // W chunks streamed by the pair
    const int32_t *trow = args.block_table + static_cast<int64_t>(b) * args.max_pages;
    // pages of this CTA's tile; a tile past the sequence (the pair's second) re-reads the
    // sequence's first page: its products are computed but never stored
    auto tile_page = [&](int i, bool *bad) -> int32_t {
        int32_t pi = 2 * tb + i;                   // page index within the sequence
        if (pi >= npages) pi = (2 * tb < npages) ? 2 * tb : 0;   // npages >= 1 here
        int32_t pg = trow[pi];
        if (pg < 0 || pg >= args.num_pages) { *bad = true; pg = 0; }
        return pg;
    };

    if (warp == 0) {
        if (ptx::elect_one()) {
            if (!kFp8) ptx::prefetch_tensormap(&map_ckv);
            ptx::prefetch_tensormap(&map_wuk);
            ptx::prefetch_tensormap(&map_wuv);
            const uint32_t ab = rank == 0 ? bar(&misc->a_full) : leader_bar(&misc->a_full);
            if (!kFp8) {
                bool bad = false;
                const int32_t pg[2] = {tile_page(0, &bad), tile_page(1, &bad)};
                if (bad) record_error(kErrDeviceBounds);
                if (rank == 0) ptx::mbar_arrive_expect_tx(ab, 2 * A_BYTES);
                for (int blk = 0; blk < CHUNKS; ++blk)
                    for (int i = 0; i < 2; ++i)
                        ptx::tma_load_3d_pair(base + OFF_A + blk * (TOK * 128) + i * (64 * 128),
                                              &map_ckv, ab, 64 * blk, 0, pg[i]);
            }
            int n = 0;
            for (; n < total; ++n) {
                const int st = n % STAGES;
                if (n >= STAGES && !wait_bounded<true>(bar(&misc->w_empty[st]),
                                                       ((n / STAGES) - 1) & 1, abort_flag,
                                                       args.timeout_ns))
                    break;
                const int32_t h = h0 + n / CHUNKS;
                const int c = n % CHUNKS;
                const uint32_t fb = rank == 0 ? bar(&misc->w_full[st]) : leader_bar(&misc->w_full[st]);
                const uint32_t sb = base + OFF_STAGE + st * STAGE_BYTES;
                if (rank == 0) ptx::mbar_arrive_expect_tx(fb, 2 * STAGE_BYTES);
                ptx::tma_load_3d_pair(sb, &map_wuk, fb, 64 * c, 64 * rank, h);
                ptx::tma_load_3d_pair(sb + WK_BYTES, &map_wuv, fb, 64 * rank, 64 * c, h);
            }
            // no copy may still be landing when the CTA exits (the abort path): the leader
            // waits for the pair's last copies
            if (rank == 0) {
                if (!kFp8) wait_bounded<true>(ab, 0, abort_flag, args.timeout_ns);
                for (int m = (n > STAGES ? n - STAGES : 0); m < n; ++m)
                    wait_bounded<true>(bar(&misc->w_full[m % STAGES]), (m / STAGES) & 1, abort_flag,
                                       args.timeout_ns);
            }
        }
    } else if (warp == 1) {
        if (rank == 0 && ptx::elect_one()) {
            bool ok = wait_bounded<true>(bar(&misc->a_full), 0, abort_flag, args.timeout_ns);
            int n = 0;
            for (int j = 0; ok && j < nh; ++j) {
                const int u = j & 1;
                if (j >= 2 && !wait_bounded<true>(bar(&misc->d_free[u]), ((j >> 1) - 1) & 1,
                                                  abort_flag, args.timeout_ns)) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                const uint32_t dk = tmem + 256u * u, dv = dk + 128u;
                for (int c = 0; c < CHUNKS; ++c, ++n) {
                    const int st = n % STAGES;
                    if (!wait_bounded<true>(bar(&misc->w_full[st]), (n / STAGES) & 1, abort_flag,
                                            args.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after();
                    const uint32_t sb = base + OFF_STAGE + st * STAGE_BYTES;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint32_t acc = (c | kk) ? 1u : 0u;
                        const uint64_t a = ptx::smem_desc(base + OFF_A + c * (TOK * 128) + kk * 32,
                                                          16, 1024, ptx::kSwizzle128B);
                        const uint64_t bk = ptx::smem_desc(sb + kk * 32, 16, 1024, ptx::kSwizzle128B);
                        ptx::mma_bf16_ss<2>(dk, a, bk, IDESC_K, acc);
                        const uint64_t bv = ptx::smem_desc(sb + WK_BYTES + kk * 2048, 64 * 128, 1024,
                                                           ptx::kSwizzle128B);
                        ptx::mma_bf16_ss<2>(dv, a, bv, IDESC_V, acc);
                    }
                    ptx::mma_commit_pair(bar(&misc->w_empty[st]), 0x3);
                }
                if (!ok) break;
                ptx::mma_commit_pair(bar(&misc->d_full[u]), 0x3);
            }
            ptx::mma_commit_pair(bar(&misc->drain), 0x1);
            wait_bounded<true>(bar(&misc->drain), 0, abort_flag, args.timeout_ns);
        }
    } else {
        const uint32_t remote_arrive_a = rank == 0 ? bar(&misc->a_full) : leader_bar(&misc->a_full);
        if (kFp8) {
            // dequantise this warp's 32 tile rows: one 512-byte row per warp load
            // (16 codes per lane), written as two swizzled 16-byte chunks per lane
            bool bad = false;
            for (int rr = 0; rr < 32; ++rr) {
                const int r = 32 * (warp - 2) + rr;
                const int32_t t = TOK * tb + r;
                uint4 lo = make_uint4(0, 0, 0, 0), hi = lo;
                if (t < L) {
                    const int32_t page = trow[t / 64];
                    if (page >= 0 && page < args.num_pages) {
                        const uint8_t *src = args.ckv8 + page * args.ckv8_page_stride +
                                             (t % 64) * args.ckv8_token_stride;
                        const float sc = args.scales[static_cast<int64_t>(page) * 64 + (t % 64)];
                        const uint4 codes = *reinterpret_cast<const uint4 *>(src + 16 * lane);
                        lo = dequant8_e4m3(codes.x, codes.y, sc);
                        hi = dequant8_e4m3(codes.z, codes.w, sc);
                    } else {
                        bad = true;
                    }
                }
                const uint32_t blk = base + OFF_A + (lane >> 2) * (TOK * 128);
                st_shared_v4(blk + sw128(r, 2 * (lane & 3)), lo.x, lo.y, lo.z, lo.w);
                st_shared_v4(blk + sw128(r, 2 * (lane & 3) + 1), hi.x, hi.y, hi.z, hi.w);
            }
            if (bad && lane == 0) record_error(kErrDeviceBounds);
            ptx::fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                if (rank == 0) ptx::mbar_arrive(remote_arrive_a);
                else ptx::mbar_arrive_cluster(remote_arrive_a);
            }
        }
        const int q4 = warp & 3;
        const int row = q4 * 32 + lane;
        const int32_t t = TOK * tb + row;
        const bool live = t < L;
        const bool store = t < rows_written;
        const uint32_t lane_base = static_cast<uint32_t>(q4 * 32) << 16;
        const uint32_t dfree = [&] {
            return rank == 0 ? ptx::smem_u32(&misc->d_free[0]) : ptx::mapa(ptx::smem_u32(&misc->d_free[0]), 0);
        }();
        for (int j = 0; j < nh; ++j) {
            const int u = j & 1;
            if (!wait_bounded<true>(bar(&misc->d_full[u]), (j >> 1) & 1, abort_flag, args.timeout_ns))
                break;
            ptx::tc_fence_after();
            const int64_t rowoff =
                ((static_cast<int64_t>(b) * args.heads + h0 + j) * args.l_pad + t) * 128;
#pragma unroll 1
            for (int part = 0; part < 2; ++part) {
                __nv_bfloat16 *dst = (part ? args.v : args.k_nope) + rowoff;
                uint32_t r[128];                    // this part's 128 columns, one wait
#pragma unroll
                for (int cch = 0; cch < 4; ++cch)
                    ptx::tmem_ld32(tmem + lane_base + 256u * u + 128u * part + 32u * cch,
                                   *reinterpret_cast<uint32_t(*)[32]>(&r[32 * cch]));
                ptx::tmem_wait_ld();
                if (store) {
                    uint4 *d4 = reinterpret_cast<uint4 *>(dst);
#pragma unroll
                    for (int q = 0; q < 16; ++q) {
                        uint4 w = make_uint4(0, 0, 0, 0);
                        if (live)
                            w = make_uint4(
                                pack_bf16x2(__uint_as_float(r[8 * q + 0]), __uint_as_float(r[8 * q + 1])),
                                pack_bf16x2(__uint_as_float(r[8 * q + 2]), __uint_as_float(r[8 * q + 3])),
                                pack_bf16x2(__uint_as_float(r[8 * q + 4]), __uint_as_float(r[8 * q + 5])),
                                pack_bf16x2(__uint_as_float(r[8 * q + 6]), __uint_as_float(r[8 * q + 7])));
                        d4[q] = w;
                    }
                }
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                const uint32_t fb = dfree + 8u * u;
                if (rank == 0) ptx::mbar_arrive(fb);
                else ptx::mbar_arrive_cluster(fb);
            }
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::cluster_sync();
    ptx::tc_fence_after();
    if (warp == 1) ptx::tmem_dealloc<2>(tmem, TMEM_COLS);
}

// ===========================================================================
// prefill_attn_kernel
// ===========================================================================
namespace pfa {
constexpr int ROWS = 128;                        // queries per CTA
constexpr int TOK = 128;                         // keys per block (two pages)
constexpr int DN = 128, DR = 64, DV = 128;
constexpr uint32_t BLK = ROWS * 128;             // one swizzled [128 x 64] bf16 block: 16 KB
constexpr uint32_t Q_BYTES = 3 * BLK;            // [q_c 0..63 | q_c 64..127 | q_r]
constexpr uint32_t K_BYTES = 3 * BLK;            // [K_nope 0..63 | K_nope 64..127 | k_R]
constexpr uint32_t V_BYTES = 2 * BLK;            // V as two MN-major [128 t x 64 e] blocks
constexpr int K_STAGES = 2, V_STAGES = 2;
constexpr uint32_t OFF_Q = 0;
constexpr uint32_t OFF_K = OFF_Q + Q_BYTES;
constexpr uint32_t OFF_V = OFF_K + K_STAGES * K_BYTES;
constexpr uint32_t OFF_MISC = OFF_V + V_STAGES * V_BYTES;
constexpr uint32_t MISC_BYTES = 1024;
constexpr uint32_t SMEM_BYTES = OFF_MISC + MISC_BYTES + 1024;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TMEM_S = 0;                   // two 128-column fp32 score buffers
constexpr uint32_t TMEM_O = 256;                 // 128 columns fp32
constexpr uint32_t TMEM_P = 384;                 // two 64-column bf16x2 probability buffers
constexpr uint32_t IDESC_QK = ptx::idesc_bf16(128, TOK, 0, 0);
constexpr uint32_t IDESC_PV = ptx::idesc_bf16(128, DV, 0, 1);
constexpr int THREADS = 192;                     // warp 0 TMA, warp 1 MMA, warps 2..5 softmax
static_assert(SMEM_BYTES <= 232448, "smem");

struct Misc {
    uint64_t q_full;
    uint64_t k_full[K_STAGES], k_empty[K_STAGES], v_full[V_STAGES], v_empty[V_STAGES];
    uint64_t s_full[2], s_free[2], p_ready[2], pv_done[2];
    uint64_t drain;
    uint32_t tmem_base;
    int32_t abort_flag;
};
static_assert(sizeof(Misc) <= MISC_BYTES, "misc");
}  // namespace pfa

struct PrefillArgs {
    const int32_t *block_table;  // [B, max_pages]
    const int32_t *seq_lens;     // [B]
    __nv_bfloat16 *out;          // [B, M, H, 128]
    float *lse;                  // [B, M, H] or null
    int64_t timeout_ns;
    int32_t batch, heads, n_q, max_pages, num_pages, l_pad, q_blocks;
    float scale, scale_log2;
};

__global__ void __launch_bounds__(pfa::THREADS, 1)
    prefill_attn_kernel(const __grid_constant__ CUtensorMap map_qc,
                        const __grid_constant__ CUtensorMap map_qr,
                        const __grid_constant__ CUtensorMap map_k,
                        const __grid_constant__ CUtensorMap map_v,
                        const __grid_constant__ CUtensorMap map_kr, const PrefillArgs args) {
    using namespace pfa;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_base = ptx::smem_u32(smem_raw);
    const uint32_t base = (raw_base + 1023u) & ~1023u;
    uint8_t *smem = smem_raw + (base - raw_base);
    pfa::Misc *misc = reinterpret_cast<pfa::Misc *>(smem + OFF_MISC);
    volatile int32_t *abort_flag = &misc->abort_flag;
    auto bar = [&](const uint64_t *b) { return ptx::smem_u32(b); };

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // heaviest query blocks (the last ones of each sequence) first
    const int32_t qb = args.q_blocks - 1 - static_cast<int32_t>(blockIdx.x);
    const int32_t h = blockIdx.y;
    const int32_t b = blockIdx.z;
    const int32_t M = args.n_q;
    const int32_t i0 = qb * ROWS;
    const int32_t L = args.seq_lens[b];
    if (L < M || static_cast<int64_t>(L) > static_cast<int64_t>(args.max_pages) * 64 ||
        L > args.l_pad) {
        if (threadIdx.x == 0 && qb == 0 && h == 0) record_error(kErrDeviceBounds);
        return;
    }
    // keys the block's last query sees: t <= L - M + min(i0 + 127, M - 1)
    const int32_t last_pos = L - M + min(i0 + ROWS - 1, M - 1);
    const int nkb = last_pos / TOK + 1;

    if (threadIdx.x == 0) {
        ptx::mbar_init(bar(&misc->q_full), 1);
        for (int i = 0; i < K_STAGES; ++i) {
            ptx::mbar_init(bar(&misc->k_full[i]), 1);
            ptx::mbar_init(bar(&misc->k_empty[i]), 1);
        }
        for (int i = 0; i < V_STAGES; ++i) {
            ptx::mbar_init(bar(&misc->v_full[i]), 1);
            ptx::mbar_init(bar(&misc->v_empty[i]), 1);
        }
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(bar(&misc->s_full[i]), 1);
            ptx::mbar_init(bar(&misc->s_free[i]), 4);
            ptx::mbar_init(bar(&misc->p_ready[i]), 4);
            ptx::mbar_init(bar(&misc->pv_done[i]), 1);
        }
        ptx::mbar_init(bar(&misc->drain), 1);
        misc->abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 1) {
        ptx::tmem_alloc<1>(bar(reinterpret_cast<uint64_t *>(&misc->tmem_base)), TMEM_COLS);
        ptx::tmem_relinquish<1>();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = misc->tmem_base;
    const int32_t bh = b * args.heads + h;

    if (warp == 0) {
        if (ptx::elect_one()) {
            ptx::prefetch_tensormap(&map_qc);
            ptx::prefetch_tensormap(&map_qr);
            ptx::prefetch_tensormap(&map_k);
            ptx::prefetch_tensormap(&map_v);
            ptx::prefetch_tensormap(&map_kr);
            const uint32_t qf = bar(&misc->q_full);
            const int32_t qrow = b * M + i0;
            ptx::mbar_arrive_expect_tx(qf, Q_BYTES);
            ptx::tma_load_3d(base + OFF_Q, &map_qc, qf, 0, h, qrow);
            ptx::tma_load_3d(base + OFF_Q + BLK, &map_qc, qf, 64, h, qrow);
            ptx::tma_load_3d(base + OFF_Q + 2 * BLK, &map_qr, qf, 0, h, qrow);
            const int32_t *trow = args.block_table + static_cast<int64_t>(b) * args.max_pages;
            const int32_t npages = (L + 63) / 64;
            bool bad = false;
            int nk = 0, nv = 0;                         // K and V blocks issued
            for (int k = 0; k < nkb; ++k) {
                const int ks = k % K_STAGES;
                if (k >= K_STAGES && !wait_bounded<false>(bar(&misc->k_empty[ks]),
                                                          ((k / K_STAGES) - 1) & 1, abort_flag,
                                                          args.timeout_ns))
                    break;
                int32_t pg[2] = {trow[2 * k], (2 * k + 1 < npages) ? trow[2 * k + 1] : -1};
                if (pg[0] < 0 || pg[0] >= args.num_pages) { bad = true; pg[0] = 0; }
                if (!(2 * k + 1 < npages)) pg[1] = pg[0];       // keys >= L are masked
                else if (pg[1] < 0 || pg[1] >= args.num_pages) { bad = true; pg[1] = 0; }
                const uint32_t kf = bar(&misc->k_full[ks]);
                const uint32_t kb = base + OFF_K + ks * K_BYTES;
                ptx::mbar_arrive_expect_tx(kf, K_BYTES);
                ptx::tma_load_3d(kb, &map_k, kf, 0, TOK * k, bh);
                ptx::tma_load_3d(kb + BLK, &map_k, kf, 64, TOK * k, bh);
                ptx::tma_load_3d(kb + 2 * BLK, &map_kr, kf, 0, 0, pg[0]);
                ptx::tma_load_3d(kb + 2 * BLK + 64 * 128, &map_kr, kf, 0, 0, pg[1]);
                nk = k + 1;
                const int vs = k % V_STAGES;
                if (k >= V_STAGES && !wait_bounded<false>(bar(&misc->v_empty[vs]),
                                                          ((k / V_STAGES) - 1) & 1, abort_flag,
                                                          args.timeout_ns))
                    break;
                const uint32_t vf = bar(&misc->v_full[vs]);
                const uint32_t vb = base + OFF_V + vs * V_BYTES;
                ptx::mbar_arrive_expect_tx(vf, V_BYTES);
                ptx::tma_load_3d(vb, &map_v, vf, 0, TOK * k, bh);
                ptx::tma_load_3d(vb + BLK, &map_v, vf, 64, TOK * k, bh);
                nv = k + 1;
            }
            if (bad) record_error(kErrDeviceBounds);
            // no copy may still be landing when the CTA exits (the abort path)
            wait_bounded<false>(qf, 0, abort_flag, args.timeout_ns);
            for (int m = (nk > K_STAGES ? nk - K_STAGES : 0); m < nk; ++m)
                wait_bounded<false>(bar(&misc->k_full[m % K_STAGES]), (m / K_STAGES) & 1,
                                    abort_flag, args.timeout_ns);
            for (int m = (nv > V_STAGES ? nv - V_STAGES : 0); m < nv; ++m)
                wait_bounded<false>(bar(&misc->v_full[m % V_STAGES]), (m / V_STAGES) & 1,
                                    abort_flag, args.timeout_ns);
        }
    } else if (warp == 1) {
        if (ptx::elect_one()) {
            auto issue_pv = [&](int kp) -> bool {
                const int s = kp & 1, vs = kp % V_STAGES;
                if (!wait_bounded<false>(bar(&misc->v_full[vs]), (kp / V_STAGES) & 1, abort_flag,
                                         args.timeout_ns) ||
                    !wait_bounded<false>(bar(&misc->p_ready[s]), (kp >> 1) & 1, abort_flag,
                                         args.timeout_ns))
                    return false;
                ptx::tc_fence_after();
                const uint32_t vb = base + OFF_V + vs * V_BYTES;
#pragma unroll
                for (int kk = 0; kk < TOK / 16; ++kk) {
                    const uint64_t bv = ptx::smem_desc(vb + kk * 2048, BLK, 1024, ptx::kSwizzle128B);
                    ptx::mma_bf16_ts<1>(tmem + TMEM_O, tmem + TMEM_P + 64u * s + 8u * kk, bv,
                                        IDESC_PV, (kp | kk) ? 1u : 0u);
                }
                ptx::mma_commit(bar(&misc->v_empty[vs]));
                ptx::mma_commit(bar(&misc->pv_done[s]));
                return true;
            };
            bool ok = wait_bounded<false>(bar(&misc->q_full), 0, abort_flag, args.timeout_ns);
            int k = 0;
            for (; ok && k < nkb; ++k) {
                const int s = k & 1, ks = k % K_STAGES;
                if (!wait_bounded<false>(bar(&misc->k_full[ks]), (k / K_STAGES) & 1, abort_flag,
                                         args.timeout_ns) ||
                    (k >= 2 && !wait_bounded<false>(bar(&misc->s_free[s]), ((k >> 1) - 1) & 1,
                                                    abort_flag, args.timeout_ns))) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                const uint32_t kb = base + OFF_K + ks * K_BYTES;
#pragma unroll
                for (int kk = 0; kk < (DN + DR) / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * BLK + (kk & 3) * 32;
                    const uint64_t a = ptx::smem_desc(base + OFF_Q + off, 16, 1024, ptx::kSwizzle128B);
                    const uint64_t bk = ptx::smem_desc(kb + off, 16, 1024, ptx::kSwizzle128B);
                    ptx::mma_bf16_ss<1>(tmem + TMEM_S + TOK * s, a, bk, IDESC_QK, kk ? 1u : 0u);
                }
                ptx::mma_commit(bar(&misc->k_empty[ks]));
                ptx::mma_commit(bar(&misc->s_full[s]));
                if (k >= 1 && !issue_pv(k - 1)) { ok = false; break; }
            }
            if (ok && nkb >= 1) issue_pv(nkb - 1);
            ptx::mma_commit(bar(&misc->drain));
            wait_bounded<false>(bar(&misc->drain), 0, abort_flag, args.timeout_ns);
        }
    } else {
        const int q4 = warp & 3;
        const int row = q4 * 32 + lane;                 // query row = TMEM lane
        const int32_t i = i0 + row;
        const bool real = i < M;
        const int32_t pos = real ? L - M + i : -1;      // last visible key; -1 sees none
        const uint32_t lane_base = static_cast<uint32_t>(q4 * 32) << 16;
        auto arrive = [&](uint64_t *bb) {
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(bar(bb));
        };
        float m_run = -INFINITY, l_run = 0.f;
        bool ok = true;
        for (int k = 0; k < nkb; ++k) {
            const int s = k & 1;
            if (!wait_bounded<false>(bar(&misc->s_full[s]), (k >> 1) & 1, abort_flag,
                                     args.timeout_ns)) {
                ok = false;
                break;
            }
            ptx::tc_fence_after();
            float v[TOK];
            {
                uint32_t sr[TOK];
#pragma unroll
                for (int c = 0; c < TOK / 32; ++c)
                    ptx::tmem_ld32(tmem + lane_base + TMEM_S + TOK * s + 32 * c,
                                   *reinterpret_cast<uint32_t(*)[32]>(&sr[32 * c]));
                ptx::tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < TOK; ++j) v[j] = __uint_as_float(sr[j]);
            }
            ptx::tc_fence_before();
            arrive(&misc->s_free[s]);

            const int32_t tok0 = TOK * k;
            if (tok0 + TOK - 1 > pos) {                 // a block on (or past) the diagonal
#pragma unroll
                for (int j = 0; j < TOK; ++j) v[j] = (tok0 + j <= pos) ? v[j] : -INFINITY;
            }
            // eight independent partial maxima / sums: one warp per SM sub-partition runs
            // this, so a single 128-long dependent chain would expose its full latency
            // (three-input max: two new keys per instruction)
            float m8[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) m8[q] = fmaxf(v[q], v[8 + q]);
#pragma unroll
            for (int j = 16; j < TOK; j += 16)
#pragma unroll
                for (int q = 0; q < 8; ++q) m8[q] = fmax3(m8[q], v[j + q], v[j + 8 + q]);
            const float mx = fmax3(fmax3(m8[0], m8[1], m8[2]), fmax3(m8[3], m8[4], m8[5]),
                                   fmaxf(m8[6], m8[7]));
            float alpha = 1.f;
            if (mx > -INFINITY &&
                (m_run == -INFINITY || (mx - m_run) * args.scale_log2 > kRescaleThreshold)) {
                alpha = (m_run == -INFINITY) ? 0.f : exp2f((m_run - mx) * args.scale_log2);
                m_run = mx;
            }
            const float mb = (m_run == -INFINITY) ? 0.f : m_run * args.scale_log2;
            // the scaling and the eight partial sums two lanes per instruction
            // (fma / add .f32x2): the loop is bound by issue slots, not by MUFU
            const float2 sc2 = make_float2(args.scale_log2, args.scale_log2);
            const float2 nmb2 = make_float2(-mb, -mb);
            float2 s2[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                            make_float2(0.f, 0.f)};
#pragma unroll
            for (int j = 0; j < TOK; j += 8)
#pragma unroll
                for (int q = 0; q < 8; q += 2) {
                    const float2 x = fma_f32x2(make_float2(v[j + q], v[j + q + 1]), sc2, nmb2);
                    v[j + q] = exp2f(x.x);
                    v[j + q + 1] = exp2f(x.y);
                    s2[q >> 1] = add_f32x2(s2[q >> 1], make_float2(v[j + q], v[j + q + 1]));
                }
            const float psum = ((s2[0].x + s2[0].y) + (s2[1].x + s2[1].y)) +
                               ((s2[2].x + s2[2].y) + (s2[3].x + s2[3].y));
            l_run = fmaf(l_run, alpha, psum);
            const bool need = (k > 0) && (alpha != 1.f);
            if (__any_sync(0xffffffffu, need)) {
                const int kp = k - 1;
                if (!wait_bounded<false>(bar(&misc->pv_done[kp & 1]), (kp >> 1) & 1, abort_flag,
                                         args.timeout_ns)) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
#pragma unroll 1
                for (int cch = 0; cch < DV / 32; ++cch) {
                    uint32_t o[32];
                    const uint32_t ta = tmem + lane_base + TMEM_O + 32 * cch;
                    ptx::tmem_ld32(ta, o);
                    ptx::tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha);
                    ptx::tmem_st32(ta, o);
                }
                ptx::tmem_wait_st();
            }
            if (k >= 2) {
                const int kp = k - 2;
                if (!wait_bounded<false>(bar(&misc->pv_done[kp & 1]), (kp >> 1) & 1, abort_flag,
                                         args.timeout_ns)) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
            }
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                uint32_t pr[32];
#pragma unroll
                for (int j = 0; j < 32; ++j) pr[j] = pack_bf16x2(v[64 * c + 2 * j], v[64 * c + 2 * j + 1]);
                ptx::tmem_st32(tmem + lane_base + TMEM_P + 64u * s + 32u * c, pr);
            }
            ptx::tmem_wait_st();
            ptx::tc_fence_before();
            arrive(&misc->p_ready[s]);
        }
        if (ok && nkb >= 1) {
            const int kl = nkb - 1;
            if (wait_bounded<false>(bar(&misc->pv_done[kl & 1]), (kl >> 1) & 1, abort_flag,
                                    args.timeout_ns)) {
                ptx::tc_fence_after();
                const float inv = (l_run > 0.f) ? 1.f / l_run : 0.f;
                __nv_bfloat16 *dst =
                    args.out + ((static_cast<int64_t>(b) * M + i) * args.heads + h) * DV;
                uint32_t o[DV];                         // four loads in flight, one wait
#pragma unroll
                for (int cch = 0; cch < DV / 32; ++cch)
                    ptx::tmem_ld32(tmem + lane_base + TMEM_O + 32 * cch,
                                   *reinterpret_cast<uint32_t(*)[32]>(&o[32 * cch]));
                ptx::tmem_wait_ld();
                if (real) {
                    uint4 *d4 = reinterpret_cast<uint4 *>(dst);
#pragma unroll
                    for (int q = 0; q < DV / 8; ++q)
                        d4[q] = make_uint4(
                            pack_bf16x2(__uint_as_float(o[8 * q + 0]) * inv, __uint_as_float(o[8 * q + 1]) * inv),
                            pack_bf16x2(__uint_as_float(o[8 * q + 2]) * inv, __uint_as_float(o[8 * q + 3]) * inv),
                            pack_bf16x2(__uint_as_float(o[8 * q + 4]) * inv, __uint_as_float(o[8 * q + 5]) * inv),
                            pack_bf16x2(__uint_as_float(o[8 * q + 6]) * inv, __uint_as_float(o[8 * q + 7]) * inv));
                }
                if (real && args.lse)
                    args.lse[(static_cast<int64_t>(b) * M + i) * args.heads + h] =
                        (l_run > 0.f) ? m_run * args.scale + logf(l_run) : -INFINITY;
            }
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    if (warp == 1) ptx::tmem_dealloc<1>(tmem, TMEM_COLS);
}

}  // namespace mla
