// The non-attention steps of the path: log-sum-exp combine of split-KV
// partials, the absorb-in projection q_c W_UK and the absorb-out projection
// o_lat W_UV, plus the timeout test hook.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>

#include "common.cuh"

namespace mla {

// (slot_base, slot_count) of sequence b under the partition plan; warp-wide.
__device__ inline void sequence_slots(const int32_t *seq_lens, int32_t batch, int32_t max_pages,
                                      int32_t n_q, int32_t tile_tokens, int64_t P, int32_t b,
                                      int64_t *slot_base, int64_t *slot_count) {
    const int lane = threadIdx.x & 31;
    bool bad = false;
    int64_t N = 0;
    for (int32_t b0 = 0; b0 < batch; b0 += 32) {
        const int32_t bb = b0 + lane;
        int64_t n = 0;
        if (bb < batch) n = tiles_of_len(clamp_len(seq_lens[bb], max_pages, n_q, &bad), tile_tokens);
        for (int o = 16; o > 0; o >>= 1) n += __shfl_xor_sync(0xffffffffu, n, o);
        N += n;
    }
    int64_t O = 0, S = 0;
    *slot_base = 0;
    *slot_count = 0;
    if (N == 0) return;
    P = parts_in_use(P, N);
    for (int32_t b0 = 0; b0 <= b; b0 += 32) {
        const int32_t bb = b0 + lane;
        int64_t n = 0;
        if (bb < batch && bb <= b)
            n = tiles_of_len(clamp_len(seq_lens[bb], max_pages, n_q, &bad), tile_tokens);
        int64_t incl = n;
        for (int o = 1; o < 32; o <<= 1) {
            const int64_t v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        const int64_t Ob = O + incl - n;
        int64_t ns = 0;
        if (n > 0) ns = part_of_tile(Ob + n - 1, N, P) - part_of_tile(Ob, N, P) + 1;
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
        O += __shfl_sync(0xffffffffu, incl, 31);
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

// grid (batch, ceil(R / 4)), 128 threads: one warp per query row.
__global__ void __launch_bounds__(128) combine_kernel(const CombineArgs a) {
    __shared__ int64_t s_base, s_count;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int32_t b = blockIdx.x;
    if (warp == 0) {
        int64_t base, cnt;
        sequence_slots(a.seq_lens, a.batch, a.max_pages, a.n_q, a.tile_tokens, a.num_parts, b,
                       &base, &cnt);
        if (lane == 0) { s_base = base; s_count = cnt; }
    }
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
    for (int c0 = 4 * lane; c0 < a.d_c; c0 += 128) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        if (m > -INFINITY) {
            for (int64_t s = 0; s < cnt; ++s) {
                const float ls = a.lse_part[(base + s) * a.rows + r];
                const float w = (ls > -INFINITY) ? __expf(ls - L) : 0.f;
                const float4 v = *reinterpret_cast<const float4 *>(
                    a.o_part + ((base + s) * a.rows + r) * a.d_c + c0);
                acc.x = fmaf(w, v.x, acc.x);
                acc.y = fmaf(w, v.y, acc.y);
                acc.z = fmaf(w, v.z, acc.z);
                acc.w = fmaf(w, v.w, acc.w);
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
// Per-head projections on CUDA cores: out[t, h, col] = sum_k x[t, h, k] W[h, k, col].
// grid (H, ceil(n_cols / 128), ceil(T / 32)), 128 threads, one output column
// per thread and 32 tokens per block; x rows staged in shared memory as fp32.
// For absorb-in (copy_rope) the block with blockIdx.y == 0 also copies q_r.
// ---------------------------------------------------------------------------
struct ProjArgs {
    const __nv_bfloat16 *x;      // [T, H, K]
    const __nv_bfloat16 *w;      // [H, K, n_cols]
    __nv_bfloat16 *out;          // [T, H, out_stride]
    const __nv_bfloat16 *rope;   // [T, H, d_rope] or null
    int32_t T, H, K, n_cols, out_stride, d_rope;
};

constexpr int kProjTok = 32;

__global__ void __launch_bounds__(128) head_proj_kernel(const ProjArgs a) {
    extern __shared__ float xs[];  // [kProjTok][K]
    const int h = blockIdx.x;
    const int col = blockIdx.y * 128 + threadIdx.x;
    const int t0 = blockIdx.z * kProjTok;
    const int nt = min(kProjTok, a.T - t0);
    for (int i = threadIdx.x; i < nt * a.K; i += 128) {
        const int t = i / a.K, k = i - t * a.K;
        xs[t * a.K + k] = __bfloat162float(a.x[(static_cast<int64_t>(t0 + t) * a.H + h) * a.K + k]);
    }
    __syncthreads();
    if (col < a.n_cols) {
        float acc[kProjTok];
#pragma unroll
        for (int t = 0; t < kProjTok; ++t) acc[t] = 0.f;
        const __nv_bfloat16 *wp = a.w + static_cast<int64_t>(h) * a.K * a.n_cols + col;
        for (int k = 0; k < a.K; ++k) {
            const float wv = __bfloat162float(wp[static_cast<int64_t>(k) * a.n_cols]);
#pragma unroll
            for (int t = 0; t < kProjTok; ++t) acc[t] = fmaf(xs[t * a.K + k], wv, acc[t]);
        }
#pragma unroll
        for (int t = 0; t < kProjTok; ++t)
            if (t < nt)
                a.out[(static_cast<int64_t>(t0 + t) * a.H + h) * a.out_stride + col] =
                    __float2bfloat16_rn(acc[t]);
    }
    if (a.rope && blockIdx.y == 0) {
        for (int i = threadIdx.x; i < nt * a.d_rope; i += 128) {
            const int t = i / a.d_rope, j = i - t * a.d_rope;
            a.out[(static_cast<int64_t>(t0 + t) * a.H + h) * a.out_stride + a.n_cols + j] =
                a.rope[(static_cast<int64_t>(t0 + t) * a.H + h) * a.d_rope + j];
        }
    }
}

// One block waits on a barrier nothing completes; the bounded wait runs out
// after timeout_ns and records kErrTimeout.
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
