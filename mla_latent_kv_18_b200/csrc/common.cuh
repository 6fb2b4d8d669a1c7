// Shared device/host helpers of the CUDA path: status codes, the device error
// word, bounded mbarrier waits and the partition plan arithmetic.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>

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

// Bounded spin until the shared-memory word at `slot` carries `tag` in its low
// 8 bits; the word is returned in *out. False after a timeout (abort raised).
__device__ __forceinline__ bool wait_word(const uint32_t *slot, uint32_t tag,
                                          volatile int32_t *abort_flag, int64_t timeout_ns,
                                          uint32_t *out) {
    const volatile uint32_t *vs = slot;
    uint32_t v = *vs;
    if ((v & 0xFFu) == tag) { *out = v; return true; }
    const uint64_t t0 = ptx::globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
        v = *vs;
        if ((v & 0xFFu) == tag) { *out = v; return true; }
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
