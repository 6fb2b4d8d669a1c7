// Shared device/host helpers of the CUDA path: status codes, the device error
// word, bounded mbarrier waits and the partition plan arithmetic.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "ptx.cuh"

namespace mla {

// Mirrors mla_status in include/mla_decode.h.
enum : int32_t {
    kOk = 0,
    kErrInvalidArg = 1,
    kErrUnsupported = 2,
    kErrCuda = 3,
    kErrDeviceBounds = 4,
    kErrTimeout = 5,
};

// First error recorded by any kernel of the library on this device.
__device__ int32_t g_device_error;

__device__ __forceinline__ void record_error(int32_t code) {
    atomicCAS(&g_device_error, 0, code);
}

// Bounded wait on phase `parity` of the barrier at shared address `bar`.
// Polls the CTA's abort flag and the global timer; after `timeout_ns` it
// records kErrTimeout, raises the abort flag and returns false.
// kClusterScope: acquire at cluster scope (needed when another CTA's arrivals
// publish generic-proxy data); otherwise CTA scope.
template <bool kClusterScope = true>
__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity,
                                             volatile int32_t *abort_flag, int64_t timeout_ns) {
    auto probe = [&] {
        return kClusterScope ? ptx::mbar_try_wait(bar, parity) : ptx::mbar_try_wait_cta(bar, parity);
    };
    if (probe()) return true;
    const uint64_t t0 = ptx::globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
        if (probe()) return true;
        if ((it & 15u) == 0u) {
            if (*abort_flag) return false;
            if (static_cast<int64_t>(ptx::globaltimer_ns() - t0) > timeout_ns) {
                record_error(kErrTimeout);
                *abort_flag = 1;
                return false;
            }
        }
    }
}

// Bounded spin until the shared-memory word at `slot` carries `tag` in its
// lowest bit; the word is returned in *out. False after a timeout (abort raised).
__device__ __forceinline__ bool wait_word(const uint32_t *slot, uint32_t tag,
                                          volatile int32_t *abort_flag, int64_t timeout_ns,
                                          uint32_t *out) {
    const volatile uint32_t *vs = slot;
    uint32_t v = *vs;
    if ((v & 1u) == tag) { *out = v; return true; }
    const uint64_t t0 = ptx::globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
        v = *vs;
        if ((v & 1u) == tag) { *out = v; return true; }
        if ((it & 15u) == 0u) {
            if (*abort_flag) return false;
            if (static_cast<int64_t>(ptx::globaltimer_ns() - t0) > timeout_ns) {
                record_error(kErrTimeout);
                *abort_flag = 1;
                return false;
            }
        }
    }
}

// Multiply written in PTX so that no flush-to-zero applies whatever the
// compile flags (subnormal products stay exact, as in the definition).
__device__ __forceinline__ float mul_rn_noftz(float a, float b) {
    float d;
    asm("mul.rn.f32 %0, %1, %2;" : "=f"(d) : "f"(a), "f"(b));
    return d;
}

// E4M3 dequantisation: bf16_rn( fp32_rn( value(code) * scale ) ). value(code)
// is exact in fp16 and fp32, so only the product and the final narrowing round.
// Two codes (the low byte is the first) to a bf16 pair (the first in the low half).
__device__ __forceinline__ uint32_t dequant2_e4m3(uint32_t two_codes, float scale) {
    const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(two_codes & 0xFFFFu),
                                                     __NV_E4M3);
    const float2 f = __half22float2(__half2(h));
    const __nv_bfloat162 v = __floats2bfloat162_rn(mul_rn_noftz(f.x, scale), mul_rn_noftz(f.y, scale));
    return *reinterpret_cast<const uint32_t *>(&v);
}

// 8 codes (two 32-bit words) to 8 bf16.
__device__ __forceinline__ uint4 dequant8_e4m3(uint32_t w0, uint32_t w1, float scale) {
    return make_uint4(dequant2_e4m3(w0, scale), dequant2_e4m3(w0 >> 16, scale), dequant2_e4m3(w1, scale),
                      dequant2_e4m3(w1 >> 16, scale));
}

// 4 codes (a 32-bit word, first code in the low byte) to 4 bf16 as two words:
// codes -> f16 pairs (exact) -> fp32 (exact) -> product (rounded once) -> bf16,
// the same arithmetic as dequant2_e4m3 in fewer instructions.
__device__ __forceinline__ uint2 dequant4_e4m3(uint32_t w, float scale) {
    uint32_t h01, h23;
    asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %2;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, lo;\n\tcvt.rn.f16x2.e4m3x2 %1, hi;\n\t}"
        : "=r"(h01), "=r"(h23)
        : "r"(w));
    float f[4];
    asm("{\n\t.reg .b16 a, b, c, d;\n\tmov.b32 {a, b}, %4;\n\tmov.b32 {c, d}, %5;\n\t"
        "cvt.f32.f16 %0, a;\n\tcvt.f32.f16 %1, b;\n\tcvt.f32.f16 %2, c;\n\tcvt.f32.f16 %3, d;\n\t}"
        : "=f"(f[0]), "=f"(f[1]), "=f"(f[2]), "=f"(f[3])
        : "r"(h01), "r"(h23));
    // products two at a time (mul.rn.f32x2, no flush-to-zero)
    float p[4];
    asm("{\n\t.reg .b64 A, B, S, D, E;\n\tmov.b64 A, {%4, %5};\n\tmov.b64 B, {%6, %7};\n\t"
        "mov.b64 S, {%8, %8};\n\tmul.rn.f32x2 D, A, S;\n\tmul.rn.f32x2 E, B, S;\n\t"
        "mov.b64 {%0, %1}, D;\n\tmov.b64 {%2, %3}, E;\n\t}"
        : "=f"(p[0]), "=f"(p[1]), "=f"(p[2]), "=f"(p[3])
        : "f"(f[0]), "f"(f[1]), "f"(f[2]), "f"(f[3]), "f"(scale));
    const __nv_bfloat162 lo = __floats2bfloat162_rn(p[0], p[1]);
    const __nv_bfloat162 hi = __floats2bfloat162_rn(p[2], p[3]);
    return make_uint2(*reinterpret_cast<const uint32_t *>(&lo), *reinterpret_cast<const uint32_t *>(&hi));
}

// max(a, b, c) in one instruction (three-input max.f32, sm_100).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// Two fp32 lanes per instruction (Blackwell's packed fp32 pipe): d = a * b + c
// and d = a + b, each lane rounded to nearest like the scalar instruction.
__device__ __forceinline__ float2 fma_f32x2(float2 a, float2 b, float2 c) {
    float2 d;
    asm("{\n\t.reg .b64 A, B, C, D;\n\tmov.b64 A, {%2, %3};\n\tmov.b64 B, {%4, %5};\n\t"
        "mov.b64 C, {%6, %7};\n\tfma.rn.f32x2 D, A, B, C;\n\tmov.b64 {%0, %1}, D;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}
__device__ __forceinline__ float2 add_f32x2(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 A, B, D;\n\tmov.b64 A, {%2, %3};\n\tmov.b64 B, {%4, %5};\n\t"
        "add.rn.f32x2 D, A, B;\n\tmov.b64 {%0, %1}, D;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}

// ---------------------------------------------------------------------------
// Partition plan. The tiles (tile_tokens tokens each) of all sequences are
// laid end to end, and before every non-empty sequence but the first the plan
// counts W = switch_cost(tile_tokens) virtual tiles: a partition that crosses
// into another sequence pays a Q load and a partial-result write there, so it
// gets correspondingly fewer real tiles. Sequence b, the j-th non-empty one,
// occupies the cost range [C_b, C_b + n_b) with C_b = O_b + W j (O_b its first
// tile); the total cost is C = N + W (NB - 1). Partition p of P owns the cost
// range [start(p), start(p+1)), start(p) = floor(p * C / P), i.e. the tiles
// whose cost position falls in it (a range inside a gap owns none). A sequence
// is covered by partitions part(C_b) .. part(C_b + n_b - 1) and gets one
// partial slot per covering partition; slots are numbered sequence-major.
// With W = 0 this is an even split of the tiles.
// ---------------------------------------------------------------------------

__host__ __device__ __forceinline__ constexpr int32_t switch_cost(int32_t tile_tokens) {
    return tile_tokens == 64 ? 8 : 3;
}

__host__ __device__ __forceinline__ int64_t part_start(int64_t p, int64_t C, int64_t P) {
    return (p * C) / P;
}

// Partition that owns cost position c (0 <= c < C): the largest p with start(p) <= c.
__host__ __device__ __forceinline__ int64_t part_of_tile(int64_t c, int64_t C, int64_t P) {
    return ((c + 1) * P + C - 1) / C - 1;
}

// Usable length of sequence b and its tile count. Lengths outside
// [n_q, max_pages * 64] are reported through `bad` and clamped.
__host__ __device__ __forceinline__ int32_t clamp_len(int32_t L, int32_t max_pages, int32_t n_q,
                                                      bool *bad) {
    const int64_t cap = static_cast<int64_t>(max_pages) * 64;
    if (L < n_q || static_cast<int64_t>(L) > cap) *bad = true;
    if (L < 0) L = 0;
    if (static_cast<int64_t>(L) > cap) L = static_cast<int32_t>(cap);
    return L;
}

__host__ __device__ __forceinline__ int64_t tiles_of_len(int32_t L, int32_t tile_tokens) {
    return (static_cast<int64_t>(L) + tile_tokens - 1) / tile_tokens;
}

// Total plan cost from the tile total N and the number NB of non-empty sequences.
__host__ __device__ __forceinline__ int64_t plan_cost(int64_t N, int64_t NB, int32_t tile_tokens) {
    return N + static_cast<int64_t>(switch_cost(tile_tokens)) * (NB > 0 ? NB - 1 : 0);
}

struct SeqCursor {
    int32_t b;          // sequence index
    int64_t cost_off;   // C_b
    int64_t slot_base;  // S_b
    int64_t total;      // C (plan cost; 0 when there is no tile)
    int64_t parts;      // partitions in use: min(num_parts, N)
};

__host__ __device__ __forceinline__ int64_t parts_in_use(int64_t num_parts, int64_t N) {
    return N < num_parts ? N : num_parts;
}

// Warp-cooperative scan: the first non-empty sequence whose cost range ends
// after cost position `ts` (the one a partition starting at ts begins with),
// with its cost offset and slot base; ts < 0 asks only for the totals. All 32
// lanes must call it; every lane gets the result.
__device__ inline SeqCursor find_sequence(const int32_t *seq_lens, int32_t batch, int32_t max_pages,
                                          int32_t n_q, int32_t tile_tokens, int64_t P,
                                          int64_t ts) {
    const int lane = threadIdx.x & 31;
    const int64_t W = switch_cost(tile_tokens);
    bool bad = false;
    int64_t N = 0, NB = 0;
    for (int32_t base = 0; base < batch; base += 32) {
        int32_t b = base + lane;
        int64_t n = 0;
        if (b < batch) n = tiles_of_len(clamp_len(seq_lens[b], max_pages, n_q, &bad), tile_tokens);
        N += __reduce_add_sync(0xffffffffu, static_cast<uint32_t>(n));
        NB += __popc(__ballot_sync(0xffffffffu, n > 0));
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) record_error(kErrDeviceBounds);
    const int64_t C = plan_cost(N, NB, tile_tokens);
    SeqCursor cur{batch, C, 0, C, parts_in_use(P, N)};
    if (N == 0 || ts < 0) return cur;
    P = cur.parts;
    int64_t CO = 0, S = 0;
    for (int32_t base = 0; base < batch; base += 32) {
        int32_t b = base + lane;
        int64_t n = 0;
        if (b < batch) n = tiles_of_len(clamp_len(seq_lens[b], max_pages, n_q, &bad), tile_tokens);
        // each non-empty sequence costs its tiles plus the gap after it, so the
        // exclusive prefix of that cost is C_b
        const int64_t w = (n > 0) ? n + W : 0;
        int64_t incl = w;
        for (int o = 1; o < 32; o <<= 1) {
            int64_t v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        const int64_t Cb = CO + incl - w;
        int64_t ns = 0;
        if (n > 0) ns = part_of_tile(Cb + n - 1, C, P) - part_of_tile(Cb, C, P) + 1;
        int64_t sincl = ns;
        for (int o = 1; o < 32; o <<= 1) {
            int64_t v = __shfl_up_sync(0xffffffffu, sincl, o);
            if (lane >= o) sincl += v;
        }
        const int64_t Sb = S + sincl - ns;
        const bool hit = (n > 0) && (Cb + n > ts);
        const unsigned m = __ballot_sync(0xffffffffu, hit);
        if (m) {
            const int src = __ffs(m) - 1;
            cur.b = __shfl_sync(0xffffffffu, b, src);
            cur.cost_off = __shfl_sync(0xffffffffu, Cb, src);
            cur.slot_base = __shfl_sync(0xffffffffu, Sb, src);
            return cur;
        }
        CO += __shfl_sync(0xffffffffu, incl, 31);
        S += __shfl_sync(0xffffffffu, sincl, 31);
    }
    return cur;
}

}  // namespace mla
