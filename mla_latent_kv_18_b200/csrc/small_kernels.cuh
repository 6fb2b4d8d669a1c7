// The non-attention steps of the path: log-sum-exp combine of split-KV
// partials, the absorb-in projection q_c W_UK and the absorb-out projection
// o_lat W_UV, plus the timeout test hook.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include <cuda.h>

#include "common.cuh"

namespace mla {

// (slot_base, slot_count) of sequence b under the partition plan (the
// cost-weighted split of common.cuh); warp-wide.
__device__ inline void sequence_slots(const int32_t *seq_lens, int32_t batch, int32_t max_pages,
                                      int32_t n_q, int32_t tile_tokens, int64_t P, int32_t b,
                                      int64_t *slot_base, int64_t *slot_count) {
    const int lane = threadIdx.x & 31;
    const int64_t W = switch_cost(tile_tokens);
    bool bad = false;
    int64_t N = 0, NB = 0;
    for (int32_t b0 = 0; b0 < batch; b0 += 32) {
        const int32_t bb = b0 + lane;
        int64_t n = 0;
        if (bb < batch) n = tiles_of_len(clamp_len(seq_lens[bb], max_pages, n_q, &bad), tile_tokens);
        NB += __popc(__ballot_sync(0xffffffffu, n > 0));
        for (int o = 16; o > 0; o >>= 1) n += __shfl_xor_sync(0xffffffffu, n, o);
        N += n;
    }
    int64_t CO = 0, S = 0;
    *slot_base = 0;
    *slot_count = 0;
    if (N == 0) return;
    const int64_t C = plan_cost(N, NB, tile_tokens);
    P = parts_in_use(P, N);
    for (int32_t b0 = 0; b0 <= b; b0 += 32) {
        const int32_t bb = b0 + lane;
        int64_t n = 0;
        if (bb < batch && bb <= b)
            n = tiles_of_len(clamp_len(seq_lens[bb], max_pages, n_q, &bad), tile_tokens);
        const int64_t w = (n > 0) ? n + W : 0;   // tiles plus the gap after the sequence
        int64_t incl = w;
        for (int o = 1; o < 32; o <<= 1) {
            const int64_t v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        const int64_t Cb = CO + incl - w;
        int64_t ns = 0;
        if (n > 0) ns = part_of_tile(Cb + n - 1, C, P) - part_of_tile(Cb, C, P) + 1;
        int64_t sincl = ns;
        for (int o = 1; o < 32; o <<= 1) {
            const int64_t v = __shfl_up_sync(0xffffffffu, sincl, o);
            if (lane >= o) sincl += v;
        }
        if (b >= b0 && b < b0 + 32) {
            const int src = b - b0;
            *slot_base = __shfl_sync(0xffffffffu, S + sincl - ns, src);
            *slot_count = __shfl_sync(0xffffffffu, ns, src);
            return;
        }
        CO += __shfl_sync(0xffffffffu, incl, 31);
        S += __shfl_sync(0xffffffffu, sincl, 31);
    }
}

// (slot_base, slot_count) of every sequence b in [b_lo, b_hi] into
// base[b - b_lo], cnt[b - b_lo] (shared memory); warp-wide, one pass.
__device__ inline void sequence_slots_range(const int32_t *seq_lens, int32_t batch, int32_t max_pages,
                                            int32_t n_q, int32_t tile_tokens, int64_t P, int32_t b_lo,
                                            int32_t b_hi, int64_t *base, int32_t *cnt) {
    const int lane = threadIdx.x & 31;
    const int64_t W = switch_cost(tile_tokens);
    bool bad = false;
    int64_t N = 0, NB = 0;
    constexpr int kCached = 8;   // per-lane tile counts kept for the second pass (batch <= 256)
    int64_t nc[kCached];
#pragma unroll
    for (int c = 0; c < kCached; ++c) {   // all loads of the cached chunks issued together
        const int32_t bb = 32 * c + lane;
        nc[c] = (bb < batch) ? tiles_of_len(clamp_len(seq_lens[bb], max_pages, n_q, &bad), tile_tokens) : 0;
    }
#pragma unroll
    for (int c = 0; c < kCached; ++c) {
        if (32 * c >= batch) break;   // uniform over the warp
        int64_t n = nc[c];
        NB += __popc(__ballot_sync(0xffffffffu, n > 0));
        for (int o = 16; o > 0; o >>= 1) n += __shfl_xor_sync(0xffffffffu, n, o);
        N += n;
    }
    for (int32_t b0 = 32 * kCached; b0 < batch; b0 += 32) {
        const int32_t bb = b0 + lane;
        int64_t n = 0;
        if (bb < batch) n = tiles_of_len(clamp_len(seq_lens[bb], max_pages, n_q, &bad), tile_tokens);
        NB += __popc(__ballot_sync(0xffffffffu, n > 0));
        for (int o = 16; o > 0; o >>= 1) n += __shfl_xor_sync(0xffffffffu, n, o);
        N += n;
    }
    for (int32_t b = b_lo + lane; b <= b_hi; b += 32) {
        base[b - b_lo] = 0;
        cnt[b - b_lo] = 0;
    }
    if (N == 0) return;
    const int64_t C = plan_cost(N, NB, tile_tokens);
    P = parts_in_use(P, N);
    int64_t CO = 0, S = 0;
    for (int32_t b0 = 0; b0 <= b_hi; b0 += 32) {
        const int32_t bb = b0 + lane;
        int64_t n = 0;
        if (bb < batch && bb <= b_hi) {
            int64_t cached = -1;
#pragma unroll
            for (int c = 0; c < kCached; ++c)
                if (b0 == 32 * c) cached = nc[c];
            n = cached >= 0 ? cached
                            : tiles_of_len(clamp_len(seq_lens[bb], max_pages, n_q, &bad), tile_tokens);
        }
        const int64_t w = (n > 0) ? n + W : 0;   // tiles plus the gap after the sequence
        int64_t incl = w;
        for (int o = 1; o < 32; o <<= 1) {
            const int64_t v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        const int64_t Cb = CO + incl - w;
        int64_t ns = 0;
        if (n > 0) ns = part_of_tile(Cb + n - 1, C, P) - part_of_tile(Cb, C, P) + 1;
        int64_t sincl = ns;
        for (int o = 1; o < 32; o <<= 1) {
            const int64_t v = __shfl_up_sync(0xffffffffu, sincl, o);
            if (lane >= o) sincl += v;
        }
        if (bb >= b_lo && bb <= b_hi) {
            base[bb - b_lo] = S + sincl - ns;
            cnt[bb - b_lo] = static_cast<int32_t>(ns);
        }
        CO += __shfl_sync(0xffffffffu, incl, 31);
        S += __shfl_sync(0xffffffffu, sincl, 31);
    }
}

struct CombineArgs {
    const float *o_part;     // [slots, R, d_c]
    const float *lse_part;   // [slots, R]
    const int32_t *seq_lens;
    __nv_bfloat16 *o_lat;    // [B, R, d_c]
    float *lse_out;          // [B, R] or null
    int32_t batch, max_pages, n_q, rows, d_c, tile_tokens, num_parts;
};

// grid (batch, ceil(R / 4)), 128 threads: one warp per query row; each lane
// keeps eight slots' loads in flight.
__global__ void __launch_bounds__(128) combine_kernel(const CombineArgs a) {
    __shared__ int64_t s_base, s_count;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int32_t b = blockIdx.x;
    ptx::grid_dep_launch();
    // the slot plan reads only the sequence lengths, which no kernel of a step
    // writes: made before waiting for the kernel before
    if (warp == 0) {
        int64_t base, cnt;
        sequence_slots(a.seq_lens, a.batch, a.max_pages, a.n_q, a.tile_tokens, a.num_parts, b,
                       &base, &cnt);
        if (lane == 0) { s_base = base; s_count = cnt; }
    }
    ptx::grid_dep_wait();   // the partials come from the kernel before
    __syncthreads();
    const int r = blockIdx.y * 4 + warp;
    if (r >= a.rows) return;
    const int64_t base = s_base, cnt = s_count;
    float m = -INFINITY;
    for (int64_t s = lane; s < cnt; s += 32) m = fmaxf(m, a.lse_part[(base + s) * a.rows + r]);
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float z = 0.f;
    if (m > -INFINITY)
        for (int64_t s = lane; s < cnt; s += 32) z += __expf(a.lse_part[(base + s) * a.rows + r] - m);
    for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
    const float L = (m > -INFINITY) ? m + __logf(z) : -INFINITY;

    __nv_bfloat16 *dst = a.o_lat + (static_cast<int64_t>(b) * a.rows + r) * a.d_c;
    const float *lse_r = a.lse_part + base * a.rows + r;
    const float *o_r = a.o_part + (base * a.rows + r) * a.d_c;
    const int64_t slot_stride = static_cast<int64_t>(a.rows) * a.d_c;
    constexpr int U = 8;   // slots in flight per thread
    for (int c0 = 4 * lane; c0 < a.d_c; c0 += 128) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        if (m > -INFINITY) {
            for (int64_t s0 = 0; s0 < cnt; s0 += U) {
                float w[U];
                float4 v[U];
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int64_t s = s0 + u;
                    w[u] = 0.f;
                    v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
                    if (s < cnt) {
                        const float ls = lse_r[s * a.rows];
                        w[u] = (ls > -INFINITY) ? __expf(ls - L) : 0.f;
                        v[u] = *reinterpret_cast<const float4 *>(o_r + s * slot_stride + c0);
                    }
                }
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    acc.x = fmaf(w[u], v[u].x, acc.x);
                    acc.y = fmaf(w[u], v[u].y, acc.y);
                    acc.z = fmaf(w[u], v[u].z, acc.z);
                    acc.w = fmaf(w[u], v[u].w, acc.w);
                }
            }
        }
        __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y);
        __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z, acc.w);
        uint2 packed;
        packed.x = *reinterpret_cast<uint32_t *>(&lo);
        packed.y = *reinterpret_cast<uint32_t *>(&hi);
        *reinterpret_cast<uint2 *>(dst + c0) = packed;
    }
    if (a.lse_out && lane == 0) a.lse_out[static_cast<int64_t>(b) * a.rows + r] = L;
}

// ---------------------------------------------------------------------------
// Per-head projections on tensor cores: out[t, h, col] = sum_k x[t, h, k] W[h, k, col]
// (absorb-in: x = q_c, W = W_UK; absorb-out: x = o_lat, W = W_UV).
// Swap-AB so the tiny token count is the MMA N: D[col, t] = W[h]^T[col, k] x^T[k, t],
// M = 128 output columns per CTA, N = NT tokens (<= 256), K in 64-wide blocks.
// W tiles are read MN-major (columns contiguous) and x tiles K-major, both by
// TMA with 128-byte swizzle; out-of-range rows/columns are zero-filled by TMA.
// grid (H, ceil(n_cols / 128), ceil(T / NT)), 128 threads: warp 0 streams the
// K blocks through a 4-stage ring, one thread of warp 1 issues the MMAs, all
// four warps drain TMEM (lane = output column) and store bf16.
// ---------------------------------------------------------------------------
// Rotary embedding of one channel pair (2p, 2p + 1) at position pos: the pair
// turns by pos * theta^(-2p / d_rope) ("MHA2MLA" page §3.2). The angle and its
// reduction to [-pi, pi] are fp64 (large positions keep their phase), the
// rotation itself fp32 ("MLA operator design" page §3: RoPE in fp32), the
// result rounded to bf16.
__device__ __forceinline__ void rope_rotate_pair(__nv_bfloat16 x0, __nv_bfloat16 x1, int32_t pos,
                                                 int pr, int d_rope, double log_theta,
                                                 __nv_bfloat16 *y0, __nv_bfloat16 *y1) {
    const double freq = exp(-2.0 * pr / d_rope * log_theta);
    const double ang = static_cast<double>(pos) * freq;
    const double two_pi = 6.283185307179586476925286766559;
    double sd, cd;
    sincos(ang - two_pi * rint(ang / two_pi), &sd, &cd);
    const float c = static_cast<float>(cd), sn = static_cast<float>(sd);
    const float f0 = __bfloat162float(x0), f1 = __bfloat162float(x1);
    *y0 = __float2bfloat16_rn(f0 * c - f1 * sn);
    *y1 = __float2bfloat16_rn(f0 * sn + f1 * c);
}

// rope_rotate_pair on a packed bf16x2 word (x0 in the low half). Out of line: its
// fp64 angle reduction is large, and the copy loop that calls it is unrolled.
__device__ __noinline__ uint32_t rope_rotate_word(uint32_t w, int32_t pos, int pr, int d_rope,
                                                  double log_theta) {
    __nv_bfloat162 x = *reinterpret_cast<const __nv_bfloat162 *>(&w);
    __nv_bfloat16 y0, y1;
    rope_rotate_pair(x.x, x.y, pos, pr, d_rope, log_theta, &y0, &y1);
    const __nv_bfloat162 y = __halves2bfloat162(y0, y1);
    return *reinterpret_cast<const uint32_t *>(&y);
}

struct ProjArgs {
    __nv_bfloat16 *out;          // [T, H, out_stride]
    const __nv_bfloat16 *rope;   // [T, H, d_rope] or null (absorb-in copies q_r)
    const int32_t *positions;    // [T] or null: rotate the copied q_r (rotary embedding)
    double log_theta;            // ln(rope_theta) when positions is set
    int64_t timeout_ns;
    int32_t T, H, K, n_cols, out_stride, d_rope, NT;
    int32_t stages;              // ring depth: min(kProjStages, K blocks)
};

constexpr int kProjStages = 4;
constexpr uint32_t kProjW = 2 * 64 * 128;   // two 64-column atoms x 64 K rows

__host__ __device__ constexpr uint32_t proj_stage_bytes(int NT) {
    return kProjW + static_cast<uint32_t>(NT) * 128;
}
__host__ __device__ constexpr uint32_t proj_smem_bytes(int NT, int stages = kProjStages) {
    return static_cast<uint32_t>(stages) * proj_stage_bytes(NT) + 1024 /* barriers */ + 1024 /* alignment */;
}

__global__ void __launch_bounds__(128) proj_tc_kernel(const __grid_constant__ CUtensorMap map_w,
                                                      const __grid_constant__ CUtensorMap map_x,
                                                      const ProjArgs a) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_base = ptx::smem_u32(smem_raw);
    const uint32_t base = (raw_base + 1023u) & ~1023u;
    uint8_t *smem = smem_raw + (base - raw_base);
    const uint32_t stage_bytes = proj_stage_bytes(a.NT);
    const int S = a.stages;   // ring depth, <= kProjStages
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + S * stage_bytes);
    uint64_t *full = bars, *empty = bars + S, *done = bars + 2 * S;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2 * S + 1);
    int32_t *abort_flag = reinterpret_cast<int32_t *>(tmem_slot + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = blockIdx.x, m0 = blockIdx.y * 128, t0 = blockIdx.z * a.NT;
    const int nkb = (a.K + 63) / 64;
    uint32_t tcols = 32;
    while (tcols < static_cast<uint32_t>(a.NT)) tcols <<= 1;

    // The weights are never written by an earlier kernel of the step, so the
    // first stages' W tiles are requested before waiting for that kernel
    // (programmatic dependent launch); the activations only after it.
    const int npre = nkb < S ? nkb : S;
    if (threadIdx.x == 0) {
        for (int i = 0; i < S; ++i) {
            ptx::mbar_init(ptx::smem_u32(&full[i]), 1);
            ptx::mbar_init(ptx::smem_u32(&empty[i]), 1);
        }
        ptx::mbar_init(ptx::smem_u32(done), 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
        for (int kb = 0; kb < npre; ++kb) {
            const uint32_t st = base + kb * stage_bytes;
            const uint32_t fb = ptx::smem_u32(&full[kb]);
            ptx::mbar_arrive_expect_tx(fb, stage_bytes);
            ptx::tma_load_3d(st, &map_w, fb, m0, kb * 64, h);
            ptx::tma_load_3d(st + 64 * 128, &map_w, fb, m0 + 64, kb * 64, h);
        }
    }
    if (warp == 1) {
        ptx::tmem_alloc<1>(ptx::smem_u32(tmem_slot), tcols);
        ptx::tmem_relinquish<1>();
    }
    ptx::grid_dep_launch();
    ptx::grid_dep_wait();   // other global memory from here on
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    volatile int32_t *abort_v = abort_flag;

    if (warp == 0) {
        if (ptx::elect_one()) {
            int kb = 0;
            for (; kb < nkb; ++kb) {
                const int s = kb % S;
                if (kb >= S &&
                    !wait_bounded(ptx::smem_u32(&empty[s]), ((kb / S) - 1) & 1, abort_v,
                                  a.timeout_ns))
                    break;
                const uint32_t st = base + s * stage_bytes;
                const uint32_t fb = ptx::smem_u32(&full[s]);
                if (kb >= npre) {   // (stages below npre: W requested before the dependency wait)
                    ptx::mbar_arrive_expect_tx(fb, stage_bytes);
                    ptx::tma_load_3d(st, &map_w, fb, m0, kb * 64, h);
                    ptx::tma_load_3d(st + 64 * 128, &map_w, fb, m0 + 64, kb * 64, h);
                }
                ptx::tma_load_3d(st + kProjW, &map_x, fb, kb * 64, h, t0);
            }
            for (int k2 = (kb > S ? kb - S : 0); k2 < kb; ++k2)
                wait_bounded(ptx::smem_u32(&full[k2 % S]), (k2 / S) & 1, abort_v,
                             a.timeout_ns);
        }
    } else if (warp == 1) {
        if (ptx::elect_one()) {
            const uint32_t idesc = ptx::idesc_bf16(128, a.NT, 1, 0);
            for (int kb = 0; kb < nkb; ++kb) {
                const int s = kb % S;
                if (!wait_bounded(ptx::smem_u32(&full[s]), (kb / S) & 1, abort_v,
                                  a.timeout_ns))
                    break;
                ptx::tc_fence_after();
                const uint32_t st = base + s * stage_bytes;
                for (int kk = 0; kk < 4; ++kk) {
                    const uint64_t ad = ptx::smem_desc(st + kk * 2048, 64 * 128, 1024, ptx::kSwizzle128B);
                    const uint64_t bd = ptx::smem_desc(st + kProjW + kk * 32, 16, 1024, ptx::kSwizzle128B);
                    ptx::mma_bf16_ss<1>(tmem, ad, bd, idesc, (kb | kk) ? 1u : 0u);
                }
                ptx::mma_commit(ptx::smem_u32(&empty[s]));
            }
            ptx::mma_commit(ptx::smem_u32(done));
        }
    } else if (a.rope && blockIdx.y == 0) {
        // warps 2 and 3, idle until the epilogue: q_r copied while the MMA runs,
        // 16 bytes (four pairs) at a time, every load of a round issued before
        // its stores (q_r rows and the q_out tail are 16-byte aligned: d_rope and
        // d_latent are multiples of 8). With positions, pair (2p, 2p + 1) turns by
        // pos * theta^(-2p / d_rope) ("MHA2MLA" page §3.2): angle and its
        // reduction to [-pi, pi] in fp64 (large positions keep their phase), the
        // rotation itself in fp32, the result rounded to bf16
        const int n8 = a.d_rope / 8;                   // 16-byte chunks per (token, head) row
        const int items = min(a.NT, a.T - t0) * n8;
        constexpr int U = 8;                           // chunks in flight per thread
        for (int i0 = threadIdx.x - 64; i0 < items; i0 += 64 * U) {
            uint4 v[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int i = i0 + 64 * u;
                if (i < items) {
                    const int t = i / n8, c8 = i - t * n8;
                    v[u] = *reinterpret_cast<const uint4 *>(
                        a.rope + (static_cast<int64_t>(t0 + t) * a.H + h) * a.d_rope + 8 * c8);
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int i = i0 + 64 * u;
                if (i >= items) continue;
                const int t = i / n8, c8 = i - t * n8;
                if (a.positions) {
                    int32_t pos = a.positions[t0 + t];
                    if (pos < 0) {
                        record_error(kErrDeviceBounds);
                        pos = 0;
                    }
                    v[u].x = rope_rotate_word(v[u].x, pos, 4 * c8 + 0, a.d_rope, a.log_theta);
                    v[u].y = rope_rotate_word(v[u].y, pos, 4 * c8 + 1, a.d_rope, a.log_theta);
                    v[u].z = rope_rotate_word(v[u].z, pos, 4 * c8 + 2, a.d_rope, a.log_theta);
                    v[u].w = rope_rotate_word(v[u].w, pos, 4 * c8 + 3, a.d_rope, a.log_theta);
                }
                *reinterpret_cast<uint4 *>(a.out + (static_cast<int64_t>(t0 + t) * a.H + h) * a.out_stride +
                                           a.n_cols + 8 * c8) = v[u];
            }
        }
    }
    // epilogue: TMEM lane = output column m0 + 32*warp + lane, column = token
    const bool ok = wait_bounded(ptx::smem_u32(done), 0, abort_v, a.timeout_ns);
    ptx::tc_fence_after();
    const int col = m0 + 32 * warp + lane;
    const int nt = min(a.NT, a.T - t0);
    if (ok) {
        for (int c0 = 0; c0 < a.NT; c0 += 32) {
            uint32_t v[32];
            ptx::tmem_ld32(tmem + (static_cast<uint32_t>(32 * warp) << 16) + c0, v);
            ptx::tmem_wait_ld();
            if (col < a.n_cols) {
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int t = c0 + j;
                    if (t < nt)
                        a.out[(static_cast<int64_t>(t0 + t) * a.H + h) * a.out_stride + col] =
                            __float2bfloat16_rn(__uint_as_float(v[j]));
                }
            }
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    if (warp == 1) ptx::tmem_dealloc<1>(tmem, tcols);
}

// One block waits on a barrier nothing completes; the bounded wait runs out
// after timeout_ns and records kErrTimeout.
// ---------------------------------------------------------------------------
// Fused combine + absorb-out: the split-KV merge followed by the per-head W_UV
// product ("MHA2MLA" page §2.1, v = c_kv W_uv applied once to the latent
// result):
//   o_lat[t, h, :] = sum_s exp(lse_s - L) o_s[t, h, :],  L = logsumexp_s lse_s
//   out[t, h, :]   = bf16(o_lat[t, h, :]) W_UV[h]        (fp32 accumulation)
// The merged row never goes back to HBM: it is rounded to bf16 straight into
// the MMA's shared-memory operand.
// grid (H * KS, ceil(T / NT)), clusters of KS CTAs along x, 128 threads. CTA q
// of head h's cluster takes latent channels [q * KC, (q + 1) * KC), KC = d_c / KS
// (64 or 128): it merges those channels of every token of its tile (same
// arithmetic and slot order as combine_kernel), streams the matching KC rows of
// W_UV[h] by TMA (MN-major, overlapped with the merge) and computes the partial
// D[col, t] = W^T[col, k] x^T[k, t] in tensor memory. The KS partial tiles are
// added in rank order over distributed shared memory, each CTA finishing
// 128 / KS output columns.
// ---------------------------------------------------------------------------
struct CombineOutArgs {
    const float *o_part;     // [slots, R, d_c]
    const float *lse_part;   // [slots, R]
    const int32_t *seq_lens;
    __nv_bfloat16 *out;      // [T, H, d_v]
    float *lse_out;          // [T, H] or null
    int64_t timeout_ns;
    int32_t batch, max_pages, n_q, H, rows, d_c, d_v, tile_tokens, num_parts, T, NT, KS;
    int32_t max_slots;       // capacity of the per-token weight rows: num_parts + 1
};

constexpr int kCoMaxNT = 64;
constexpr int kCoMaxSlots = 160;   // partial slots per sequence (num_parts + 1 at most)
// Shared memory of a combine_out_kernel CTA. The partial D tile of the K-split
// ([t][col] fp32, NT * 512 bytes) reuses the W_UV rows once the MMA has read
// them, and the weight rows hold max_slots entries, so that five CTAs fit on an
// SM (the grid has H * KS CTAs per 16 or 32 tokens).
constexpr uint32_t kCoFourPerSmSmem = 49152;   // above a fifth of the SM's 228 KB, within a quarter
__host__ __device__ constexpr uint32_t co_smem_bytes(int KC, int NT, int max_slots) {
    return static_cast<uint32_t>(KC / 64) * 16384u            // W_UV rows: two 64-column atoms per K block
           + static_cast<uint32_t>(KC / 64) * NT * 128u        // merged rows (bf16, K-major, swizzled)
           + static_cast<uint32_t>(NT) * max_slots * 4u        // merge weights [t][slot]
           + static_cast<uint32_t>(NT) * 16u                   // per token: first slot, count, row
           + static_cast<uint32_t>(NT) * 16u                   // per sequence: first slot, count
           + 128u /* barriers */ + 1024u /* alignment */;
}

__global__ void __launch_bounds__(128) combine_out_kernel(const __grid_constant__ CUtensorMap map_w,
                                                          const CombineOutArgs a) {
    extern __shared__ uint8_t co_smem_raw[];
    const uint32_t raw_base = ptx::smem_u32(co_smem_raw);
    const uint32_t base = (raw_base + 1023u) & ~1023u;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int KS = a.KS, NT = a.NT;
    const uint32_t q = (KS > 1) ? ptx::cluster_ctarank() : 0u;
    const int h = blockIdx.x / KS;
    const int t0 = blockIdx.y * NT;
    const int KC = a.d_c / KS;
    const int KB = KC / 64;
    const int nt = min(NT, a.T - t0);
    const uint32_t w_s = base;
    const uint32_t x_s = w_s + KB * 16384u;
    const uint32_t part_s = w_s;   // the partial D tile, once the MMA has read the W_UV rows
    const uint32_t wts_s = x_s + KB * NT * 128u;
    const int MS = a.max_slots;
    const uint32_t tok_s = wts_s + NT * MS * 4u;
    const uint32_t seq_s = tok_s + NT * 16u;
    const uint32_t bar_s = seq_s + NT * 16u;
    int64_t *seq_base = reinterpret_cast<int64_t *>(co_smem_raw + (seq_s - raw_base));
    int32_t *seq_cnt = reinterpret_cast<int32_t *>(co_smem_raw + (seq_s - raw_base) + NT * 8);
    float *wts = reinterpret_cast<float *>(co_smem_raw + (wts_s - raw_base));
    int64_t *tok_base = reinterpret_cast<int64_t *>(co_smem_raw + (tok_s - raw_base));
    int32_t *tok_cnt = reinterpret_cast<int32_t *>(co_smem_raw + (tok_s - raw_base) + NT * 8);
    int32_t *tok_row = reinterpret_cast<int32_t *>(co_smem_raw + (tok_s - raw_base) + NT * 12);
    uint8_t *bar_p = co_smem_raw + (bar_s - raw_base);
    const uint32_t wfull = bar_s, done = bar_s + 8;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar_p + 16);
    int32_t *abort_flag = reinterpret_cast<int32_t *>(bar_p + 20);
    uint32_t tcols = 32;
    while (tcols < static_cast<uint32_t>(NT)) tcols <<= 1;

    ptx::grid_dep_launch();
    if (threadIdx.x == 0) {
        ptx::mbar_init(wfull, 1);
        ptx::mbar_init(done, 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
        // W_UV[h] rows [q * KC, (q + 1) * KC): never written by an earlier kernel
        // of the step, so requested before waiting for it; lands during the merge
        ptx::mbar_arrive_expect_tx(wfull, KB * 16384u);
        for (int kb = 0; kb < KB; ++kb) {
            const int k0 = static_cast<int>(q) * KC + kb * 64;
            ptx::tma_load_3d(w_s + kb * 16384u, &map_w, wfull, 0, k0, h);
            ptx::tma_load_3d(w_s + kb * 16384u + 8192u, &map_w, wfull, 64, k0, h);
        }
    }
    // the slots of the tile's sequences: the plan reads only the sequence
    // lengths, which no kernel of a step writes, so it is made before the wait
    const int32_t b_lo = t0 / a.n_q, b_hi = (t0 + nt - 1) / a.n_q;   // at most NT sequences
    if (warp == 0)
        sequence_slots_range(a.seq_lens, a.batch, a.max_pages, a.n_q, a.tile_tokens, a.num_parts,
                             b_lo, b_hi, seq_base, seq_cnt);
    ptx::grid_dep_wait();   // other global memory from here on
    if (warp == 1) {
        ptx::tmem_alloc<1>(ptx::smem_u32(tmem_slot), tcols);
        ptx::tmem_relinquish<1>();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    volatile int32_t *abort_v = abort_flag;

    // ---- merge, phase 1: eight threads per token find L and the weights
    // exp(lse_s - L) with the same arithmetic and the same addition tree as
    // combine_kernel (the slots were found above; the barrier above publishes them)
    for (int tt = threadIdx.x >> 3; tt < NT; tt += 16) {
        const int sub = threadIdx.x & 7;
        const bool live = tt < nt;
        int64_t sbase = 0;
        int cnt = 0, r = 0;
        if (live) {
            const int t = t0 + tt;
            const int32_t b = t / a.n_q;
            r = (t - b * a.n_q) * a.H + h;
            sbase = seq_base[b - b_lo];
            cnt = seq_cnt[b - b_lo];
        }
        const float *lse_r = a.lse_part + sbase * a.rows + r;
        // thread sub stands for lanes sub, sub + 8, sub + 16, sub + 24 of a warp
        // that strides the slots by 32; the first 32 slots' values stay in
        // registers (one load round), later ones are read again
        float lv[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int s = sub + 8 * j;
            lv[j] = (s < cnt) ? lse_r[static_cast<int64_t>(s) * a.rows] : -INFINITY;
        }
        float mv[4] = {lv[0], lv[1], lv[2], lv[3]};
#pragma unroll
        for (int j = 0; j < 4; ++j)
            for (int s = sub + 8 * j + 32; s < cnt; s += 32)
                mv[j] = fmaxf(mv[j], lse_r[static_cast<int64_t>(s) * a.rows]);
        float m = fmaxf(fmaxf(mv[0], mv[2]), fmaxf(mv[1], mv[3]));
        for (int o = 4; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        float zv[4] = {0.f, 0.f, 0.f, 0.f};
        if (m > -INFINITY) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                if (sub + 8 * j < cnt) zv[j] = __expf(lv[j] - m);
                for (int s = sub + 8 * j + 32; s < cnt; s += 32)
                    zv[j] += __expf(lse_r[static_cast<int64_t>(s) * a.rows] - m);
            }
        }
        // the 32-lane xor tree: +16, +8 locally, then +4, +2, +1 across the 8 threads
        float z = (zv[0] + zv[2]) + (zv[1] + zv[3]);
        for (int o = 4; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
        const float L = (m > -INFINITY) ? m + __logf(z) : -INFINITY;
        if (live && a.lse_out && q == 0 && sub == 0)
            a.lse_out[static_cast<int64_t>(t0 + tt) * a.H + h] = L;
        if (m == -INFINITY || cnt > MS) cnt = 0;   // nothing to merge (the host caps the slots)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int s = sub + 8 * j;
            if (s < cnt) wts[tt * MS + s] = (lv[j] > -INFINITY) ? __expf(lv[j] - L) : 0.f;
        }
        for (int s = sub + 32; s < cnt; s += 8) {
            const float ls = lse_r[static_cast<int64_t>(s) * a.rows];
            wts[tt * MS + s] = (ls > -INFINITY) ? __expf(ls - L) : 0.f;
        }
        if (sub == 0) {
            tok_base[tt] = sbase;
            tok_cnt[tt] = cnt;
            tok_row[tt] = r;
        }
    }
    __syncthreads();
    // ---- merge, phase 2: items (token, 4 channels), all loads of a slot step
    // issued together; slots are added in order, as in combine_kernel
    {
        const int chunks = KC / 4;
        constexpr int IT = 4;   // items per thread and round (NT * chunks / 512 rounds)
        const int64_t slot_stride = static_cast<int64_t>(a.rows) * a.d_c;
        for (int i0 = threadIdx.x; i0 < NT * chunks; i0 += IT * 128) {
            float4 acc[IT];
            const float *src[IT];
            int cnt_i[IT], tt_i[IT];
            int maxc = 0;
#pragma unroll
            for (int u = 0; u < IT; ++u) {
                acc[u] = make_float4(0.f, 0.f, 0.f, 0.f);
                const int i = i0 + u * 128;
                tt_i[u] = i / chunks;
                const bool live = i < NT * chunks;
                cnt_i[u] = live ? tok_cnt[tt_i[u]] : 0;
                src[u] = live ? a.o_part + (tok_base[tt_i[u]] * a.rows + tok_row[tt_i[u]]) * a.d_c +
                                    q * KC + 4 * (i - tt_i[u] * chunks)
                              : a.o_part;
                maxc = max(maxc, cnt_i[u]);
            }
            constexpr int SS = 4;   // slots per step
            for (int s = 0; s < maxc; s += SS) {
                float4 v[IT][SS];
                float w[IT][SS];
#pragma unroll
                for (int u = 0; u < IT; ++u)
#pragma unroll
                    for (int e = 0; e < SS; ++e) {
                        const bool on = s + e < cnt_i[u];
                        v[u][e] = on ? *reinterpret_cast<const float4 *>(src[u] + (s + e) * slot_stride)
                                     : make_float4(0.f, 0.f, 0.f, 0.f);
                        w[u][e] = on ? wts[tt_i[u] * MS + s + e] : 0.f;
                    }
#pragma unroll
                for (int u = 0; u < IT; ++u)
#pragma unroll
                    for (int e = 0; e < SS; ++e) {
                        if (s + e < cnt_i[u]) {
                            acc[u].x = fmaf(w[u][e], v[u][e].x, acc[u].x);
                            acc[u].y = fmaf(w[u][e], v[u][e].y, acc[u].y);
                            acc[u].z = fmaf(w[u][e], v[u][e].z, acc[u].z);
                            acc[u].w = fmaf(w[u][e], v[u][e].w, acc[u].w);
                        }
                    }
            }
#pragma unroll
            for (int u = 0; u < IT; ++u) {   // bf16 into the K-major, 128-byte-swizzled operand tile
                const int i = i0 + u * 128;
                if (i >= NT * chunks) continue;
                const int c_loc = 4 * (i - tt_i[u] * chunks);
                __nv_bfloat162 lo = __floats2bfloat162_rn(acc[u].x, acc[u].y);
                __nv_bfloat162 hi = __floats2bfloat162_rn(acc[u].z, acc[u].w);
                const int kb = c_loc >> 6, within = c_loc & 63;
                const uint32_t addr = x_s + kb * NT * 128u + sw128(tt_i[u], within >> 3) + ((within & 7) >> 2) * 8u;
                asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(addr),
                             "r"(*reinterpret_cast<uint32_t *>(&lo)), "r"(*reinterpret_cast<uint32_t *>(&hi))
                             : "memory");
            }
        }
    }
    ptx::fence_proxy_async_smem();
    __syncthreads();

    // ---- tensor cores: D[col, t] = sum_k W[k, col] x[t, k] over this CTA's KC rows
    if (warp == 1 && ptx::elect_one()) {
        if (wait_bounded<false>(wfull, 0, abort_v, a.timeout_ns)) {
            ptx::tc_fence_after();
            const uint32_t idesc = ptx::idesc_bf16(128, NT, 1, 0);
            for (int kb = 0; kb < KB; ++kb) {
                for (int kk = 0; kk < 4; ++kk) {
                    const uint64_t ad = ptx::smem_desc(w_s + kb * 16384u + kk * 2048u, 64 * 128, 1024,
                                                       ptx::kSwizzle128B);
                    const uint64_t bd = ptx::smem_desc(x_s + kb * NT * 128u + kk * 32u, 16, 1024,
                                                       ptx::kSwizzle128B);
                    ptx::mma_bf16_ss<1>(tmem, ad, bd, idesc, (kb | kk) ? 1u : 0u);
                }
            }
        }
        ptx::mma_commit(done);
    }
    const bool ok = wait_bounded<false>(done, 0, abort_v, a.timeout_ns) && !*abort_v;
    ptx::tc_fence_after();
    const int col = 32 * warp + lane;   // TMEM lane = output column
    if (KS == 1) {
        if (ok) {
            for (int c0 = 0; c0 < NT; c0 += 32) {
                uint32_t v[32];
                ptx::tmem_ld32(tmem + (static_cast<uint32_t>(32 * warp) << 16) + c0, v);
                ptx::tmem_wait_ld();
                if (col < a.d_v) {
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const int t = c0 + j;
                        if (t < nt)
                            a.out[(static_cast<int64_t>(t0 + t) * a.H + h) * a.d_v + col] =
                                __float2bfloat16_rn(__uint_as_float(v[j]));
                    }
                }
            }
        }
    } else {
        // partial tile to shared memory as [t][col], then the rank-ordered sum
        for (int c0 = 0; c0 < NT; c0 += 32) {
            uint32_t v[32];
            ptx::tmem_ld32(tmem + (static_cast<uint32_t>(32 * warp) << 16) + c0, v);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const int t = c0 + j;
                if (t < NT) {
                    const float val = ok ? __uint_as_float(v[j]) : 0.f;
                    asm volatile("st.shared.f32 [%0], %1;" ::"r"(part_s + (t * 128u + col) * 4u), "f"(val)
                                 : "memory");
                }
            }
        }
        ptx::cluster_sync();
        const int cw = 128 / KS;   // output columns finished by this CTA
        const int c4 = cw / 4;     // 4-column groups per token
        for (int idx = threadIdx.x; idx < nt * c4; idx += 128) {
            const int t = idx / c4, cl = static_cast<int>(q) * cw + 4 * (idx - t * c4);
            const uint32_t off = part_s + (t * 128u + cl) * 4u;
            float4 pr[8];   // KS <= 8: every rank's partial requested before any is added
#pragma unroll
            for (int rk = 0; rk < 8; ++rk)
                if (rk < KS) pr[rk] = ptx::ld_shared_cluster_v4(ptx::mapa(off, rk));
            float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int rk = 0; rk < 8; ++rk)
                if (rk < KS) {
                    sum.x += pr[rk].x;
                    sum.y += pr[rk].y;
                    sum.z += pr[rk].z;
                    sum.w += pr[rk].w;
                }
            if (cl < a.d_v) {   // d_v is a multiple of 8: the group is all in or all out
                __nv_bfloat162 lo = __floats2bfloat162_rn(sum.x, sum.y);
                __nv_bfloat162 hi = __floats2bfloat162_rn(sum.z, sum.w);
                uint2 packed;
                packed.x = *reinterpret_cast<uint32_t *>(&lo);
                packed.y = *reinterpret_cast<uint32_t *>(&hi);
                *reinterpret_cast<uint2 *>(a.out + (static_cast<int64_t>(t0 + t) * a.H + h) * a.d_v + cl) = packed;
            }
        }
        ptx::cluster_sync();   // peers read this CTA's tile until here
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    if (warp == 1) ptx::tmem_dealloc<1>(tmem, tcols);
}

// ---------------------------------------------------------------------------
// Debug gather: the page lookup of the decode kernels (token t of sequence b
// is row t % 64 of page block_table[b][t / 64], "MLA operator design" page §3)
// through a TMA pool descriptor like theirs, written out densely.
// grid (batch, max_pages), 128 threads, dynamic smem 64 x width x 2 bytes:
// CTA (b, pg) loads page pg of sequence b as width / box_ch boxes of
// [64 tokens x box_ch channels] and copies its valid tokens to out.
// ---------------------------------------------------------------------------
struct GatherArgs {
    const int32_t *block_table;  // [B, max_pages]
    const int32_t *seq_lens;     // [B]
    __nv_bfloat16 *out;          // [B, max_len, width]
    int64_t timeout_ns;
    int32_t batch, max_pages, num_pages, width, box_ch, max_len;
};

__global__ void __launch_bounds__(128) gather_kernel(const __grid_constant__ CUtensorMap map,
                                                     const GatherArgs a) {
    extern __shared__ __align__(128) uint8_t gather_smem[];
    __shared__ __align__(8) uint64_t bar;
    __shared__ int32_t abort_flag;
    const int32_t b = blockIdx.x, pg = blockIdx.y;
    const int32_t L = a.seq_lens[b];
    if (L < 0 || L > a.max_len || static_cast<int64_t>(L) > static_cast<int64_t>(a.max_pages) * 64) {
        if (threadIdx.x == 0 && pg == 0) record_error(kErrDeviceBounds);
        return;
    }
    if (static_cast<int64_t>(pg) * 64 >= L) return;   // entries past the last page are not read
    const int32_t page = a.block_table[static_cast<int64_t>(b) * a.max_pages + pg];
    if (page < 0 || page >= a.num_pages) {
        if (threadIdx.x == 0) record_error(kErrDeviceBounds);
        return;
    }
    const uint32_t base = ptx::smem_u32(gather_smem);
    const uint32_t bb = ptx::smem_u32(&bar);
    const int nbox = a.width / a.box_ch;
    if (threadIdx.x == 0) {
        ptx::mbar_init(bb, 1);
        abort_flag = 0;
        ptx::fence_mbar_init();
        ptx::mbar_arrive_expect_tx(bb, static_cast<uint32_t>(64 * a.width * 2));
        for (int j = 0; j < nbox; ++j)
            ptx::tma_load_3d(base + static_cast<uint32_t>(j * 64 * a.box_ch * 2), &map, bb,
                             j * a.box_ch, 0, page);
    }
    __syncthreads();
    if (!wait_bounded<false>(bb, 0, &abort_flag, a.timeout_ns)) return;
    const int n = min(64, L - pg * 64);
    const int c8n = a.width / 8;
    __nv_bfloat16 *dst = a.out + (static_cast<int64_t>(b) * a.max_len + static_cast<int64_t>(pg) * 64) * a.width;
    for (int idx = threadIdx.x; idx < n * c8n; idx += blockDim.x) {
        const int t = idx / c8n, c = (idx - t * c8n) * 8;
        const int j = c / a.box_ch, cin = c - j * a.box_ch;
        const uint4 v = *reinterpret_cast<const uint4 *>(gather_smem + (static_cast<int64_t>(j) * 64 + t) * a.box_ch * 2 + cin * 2);
        *reinterpret_cast<uint4 *>(dst + static_cast<int64_t>(t) * a.width + c) = v;
    }
}

__global__ void wait_timeout_kernel(int64_t timeout_ns) {
    __shared__ __align__(8) uint64_t b;
    __shared__ int32_t abort_flag;
    if (threadIdx.x == 0) {
        ptx::mbar_init(ptx::smem_u32(&b), 1);
        abort_flag = 0;
    }
    __syncthreads();
    if (threadIdx.x == 0) wait_bounded(ptx::smem_u32(&b), 0, &abort_flag, timeout_ns);
}

}  // namespace mla

namespace mla {

// ---------------------------------------------------------------------------
// Cache write: new tokens' latent c_KV and decoupled RoPE key k_R into the
// paged pools, with the rotary embedding applied to k_R on the way in
// ("MLA operator design" page §3: page_size 64, RoPE in fp32; "MHA2MLA" page
// §3.2: rope_theta). One warp per token: the c_KV row is a 16-byte-vector
// copy, each lane rotates one channel pair of k_R at a time.
// ---------------------------------------------------------------------------
struct AppendArgs {
    const __nv_bfloat16 *ckv_new;   // [T, d_c]
    const __nv_bfloat16 *kr_new;    // [T, d_r] (unrotated)
    const int32_t *seq_ids;         // [T]
    const int32_t *positions;       // [T]
    const int32_t *block_table;     // [batch, max_pages]
    __nv_bfloat16 *ckv;             // pool base (bf16 cache), or null
    uint8_t *ckv8;                  // pool base (E4M3 cache), or null
    float *scales;                  // [pages, 64] with the E4M3 cache
    __nv_bfloat16 *kr;              // pool base
    int64_t ckv_page_stride, ckv_token_stride, kr_page_stride, kr_token_stride;   // elements
    double log_theta;               // ln(rope_theta); rotate only if rotate != 0
    int32_t T, d_c, d_r, batch, max_pages, num_pages, rotate;
};

__global__ void __launch_bounds__(256) append_kv_kernel(const AppendArgs a) {
    const int lane = threadIdx.x & 31;
    const int64_t t = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
    if (t >= a.T) return;
    const int32_t b = a.seq_ids[t], pos = a.positions[t];
    bool ok = b >= 0 && b < a.batch && pos >= 0 &&
              static_cast<int64_t>(pos) < static_cast<int64_t>(a.max_pages) * 64;
    int32_t page = 0;
    if (ok) {
        page = a.block_table[static_cast<int64_t>(b) * a.max_pages + pos / 64];
        ok = page >= 0 && page < a.num_pages;
    }
    if (!ok) {                       // uniform over the warp
        if (lane == 0) record_error(kErrDeviceBounds);
        return;
    }
    const int slot = pos % 64;
    const uint4 *src = reinterpret_cast<const uint4 *>(a.ckv_new + t * a.d_c);
    if (a.ckv8) {
        // E4M3 with one fp32 scale per token: amax over the row, then
        // inv = 448 / amax, code = E4M3_rn_satfinite(x * inv), scale = amax / 448,
        // all with IEEE-rounded fp32 operations
        float amax = 0.f;
        for (int i = lane; i < a.d_c / 8; i += 32) {
            const uint4 v = src[i];
            const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&v);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float2 f = __bfloat1622float2(h[q]);
                amax = fmaxf(amax, fmaxf(fabsf(f.x), fabsf(f.y)));
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        const float inv = amax > 0.f ? __fdiv_rn(448.f, amax) : 1.f;
        uint8_t *dst8 = a.ckv8 + page * a.ckv_page_stride + slot * a.ckv_token_stride;
        for (int i = lane; i < a.d_c / 8; i += 32) {
            const uint4 v = src[i];
            const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&v);
            uint32_t w[2];
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                const float2 f0 = __bfloat1622float2(h[2 * q]), f1 = __bfloat1622float2(h[2 * q + 1]);
                const uint32_t c0 = __nv_cvt_float_to_fp8(__fmul_rn(f0.x, inv), __NV_SATFINITE, __NV_E4M3);
                const uint32_t c1 = __nv_cvt_float_to_fp8(__fmul_rn(f0.y, inv), __NV_SATFINITE, __NV_E4M3);
                const uint32_t c2 = __nv_cvt_float_to_fp8(__fmul_rn(f1.x, inv), __NV_SATFINITE, __NV_E4M3);
                const uint32_t c3 = __nv_cvt_float_to_fp8(__fmul_rn(f1.y, inv), __NV_SATFINITE, __NV_E4M3);
                w[q] = c0 | (c1 << 8) | (c2 << 16) | (c3 << 24);
            }
            *reinterpret_cast<uint2 *>(dst8 + 8 * i) = make_uint2(w[0], w[1]);
        }
        if (lane == 0) a.scales[static_cast<int64_t>(page) * 64 + slot] = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
    } else {
        uint4 *dst = reinterpret_cast<uint4 *>(a.ckv + page * a.ckv_page_stride + slot * a.ckv_token_stride);
        for (int i = lane; i < a.d_c / 8; i += 32) dst[i] = src[i];
    }
    const __nv_bfloat16 *r = a.kr_new + t * a.d_r;
    __nv_bfloat16 *rd = a.kr + page * a.kr_page_stride + slot * a.kr_token_stride;
    for (int p = lane; p < a.d_r / 2; p += 32) {
        if (a.rotate) {
            rope_rotate_pair(r[2 * p], r[2 * p + 1], pos, p, a.d_r, a.log_theta, &rd[2 * p],
                             &rd[2 * p + 1]);
        } else {
            rd[2 * p] = r[2 * p];
            rd[2 * p + 1] = r[2 * p + 1];
        }
    }
}

}  // namespace mla

namespace mla {

// ---------------------------------------------------------------------------
// Dequantising gather of the E4M3 latent cache (the quantised cache gather of
// the "MLA operator design" page, introduction and §5, with 16-byte loads):
//   out[b, t, c] = bf16( value(code[b, t, c]) * scale[b, t] )   for t < seq_lens[b]
// One warp per (sequence, token) row; each lane loads 16 codes (16 bytes) and
// writes 32 bytes of bf16.
// ---------------------------------------------------------------------------
struct GatherFp8Args {
    const uint8_t *ckv8;            // pool base
    const float *scales;            // [pages, 64]
    const int32_t *block_table;     // [batch, max_pages]
    const int32_t *seq_lens;        // [batch]
    __nv_bfloat16 *out;             // [batch, max_len, width]
    int64_t page_stride, token_stride;   // bytes
    int32_t width, num_pages, max_pages, batch, max_len;
};

__global__ void __launch_bounds__(256) gather_dequant_fp8_kernel(const GatherFp8Args a) {
    const int lane = threadIdx.x & 31;
    const int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
    if (row >= static_cast<int64_t>(a.batch) * a.max_len) return;
    const int32_t b = static_cast<int32_t>(row / a.max_len);
    const int32_t t = static_cast<int32_t>(row - static_cast<int64_t>(b) * a.max_len);
    const int32_t L = a.seq_lens[b];
    if (L < 0 || L > a.max_len || static_cast<int64_t>(L) > static_cast<int64_t>(a.max_pages) * 64) {
        if (t == 0 && lane == 0) record_error(kErrDeviceBounds);
        return;
    }
    if (t >= L) return;
    const int32_t page = a.block_table[static_cast<int64_t>(b) * a.max_pages + t / 64];
    if (page < 0 || page >= a.num_pages) {
        if (lane == 0) record_error(kErrDeviceBounds);
        return;
    }
    const uint8_t *src = a.ckv8 + page * a.page_stride + (t % 64) * a.token_stride;
    const float scale = a.scales[static_cast<int64_t>(page) * 64 + (t % 64)];
    __nv_bfloat16 *dst = a.out + row * a.width;
    for (int i = lane; i < a.width / 16; i += 32) {
        const uint4 codes = *reinterpret_cast<const uint4 *>(src + 16 * i);
        reinterpret_cast<uint4 *>(dst + 16 * i)[0] = dequant8_e4m3(codes.x, codes.y, scale);
        reinterpret_cast<uint4 *>(dst + 16 * i)[1] = dequant8_e4m3(codes.z, codes.w, scale);
    }
}

}  // namespace mla
