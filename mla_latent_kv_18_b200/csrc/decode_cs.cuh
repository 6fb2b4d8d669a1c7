// Split-KV MLA decode, d_c = 512 / d_R = 64, on a CTA pair that splits the
// latent channels ("MLA operator design" page §4 path B; "MHA2MLA" page §2.1).
//
// Each CTA of a two-CTA cluster (two SMs) owns one half of the channels of
// every cached token: CTA h loads c_KV channels [256h, 256h + 256) and k_R
// channels [32h, 32h + 32) of each 64-token page, so each byte of the cache is
// read from L2 by exactly one SM. Per tile, with cta_group::1 MMAs and M = 128
// query rows:
//   S_h = Q[:, own channels] [c_KV | k_R][:, own channels]^T   (partial scores)
//   the two partials are exchanged over distributed shared memory (st.async),
//   and both CTAs form S = S_0 + S_1 (the same fp32 sum in either order), run
//   the same fp32 online softmax on all 128 rows, and write P (bf16);
//   O_h += P c_KV[:, own channels]                              (value product)
// so O_h = O[:, 256h : 256h + 256] stays in this CTA's tensor memory and the
// partial result of a segment is O_h / l, lse = m * scale + ln l, written by
// each CTA for its channels (lse by CTA 0).
//
// Tensor memory (512 columns): O_h 256, two 64-column score buffers, Q's
// latent channels of this half (256 bf16 = 128 columns, the A operand of the
// QK^T MMA). Shared memory: a three-slot ring of 36 KB KV half-pages, two
// 32 KB buffers receiving the peer's partial scores, two P buffers, Q's RoPE
// channels (the A operand of the last two K steps).
//
// Warp roles (14 warps): warp 0 TMA producer; warp 1 MMA issuer (one thread);
// warps 2..9 softmax (two warps per tensor-memory lane quadrant, each row held
// by two threads of those warps, 32 tokens and 128 O columns each); warps
// 10..13 send this CTA's partial scores to the peer and load Q.
//
// Rows past a sequence's end in its last page are cleared in shared memory
// before the value product reads them, so whatever bits an unwritten or
// recycled page slot holds never reach a result. Every wait is bounded.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda.h>

#include "common.cuh"
#include "decode.cuh"

namespace mla {
namespace cs {
constexpr int DC = 512, DR = 64, D = DC + DR;
constexpr int TOK = 64;                               // tokens per tile (one page)
constexpr int ROWS = 128;                             // query rows (M)
constexpr int HC = DC / 2, HR = DR / 2;               // this CTA's latent / RoPE channels
constexpr int NST = 3;                                // KV ring depth
constexpr int THREADS = 448;                          // 14 warps
constexpr int SMX0 = 2;                               // first softmax warp
constexpr int SND0 = 10;                              // first sender warp
constexpr uint32_t BLK = TOK * 128;                   // [64 tok x 64 ch] bf16, 128-byte swizzle
constexpr uint32_t RBLK = TOK * 64;                   // [64 tok x 32 ch] bf16, 64-byte swizzle
constexpr uint32_t STAGE = 4 * BLK + RBLK;            // 36864
constexpr uint32_t XBUF = ROWS * TOK * 4;             // [128 x 64] fp32 partial scores
constexpr uint32_t PBUF = ROWS * 128;                 // [128 x 64] bf16, 128-byte swizzle
constexpr uint32_t QROPE = ROWS * 64;                 // [128 x 32] bf16, 64-byte swizzle
constexpr uint32_t OFF_KV = 0;
constexpr uint32_t OFF_X = OFF_KV + NST * STAGE;      // 110592
constexpr uint32_t OFF_P = OFF_X + 2 * XBUF;          // 176128
constexpr uint32_t OFF_QR = OFF_P + 2 * PBUF;         // 208896
constexpr uint32_t OFF_MISC = OFF_QR + QROPE;         // 217088
constexpr uint32_t MISC_BYTES = 7168;
constexpr uint32_t SMEM_BYTES = OFF_MISC + MISC_BYTES;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TMEM_O = 0;                        // 256 columns
constexpr uint32_t TMEM_S = 256;                      // two 64-column score buffers
constexpr uint32_t TMEM_Q = 384;                      // 128 columns: Q latent channels, bf16 pairs
constexpr uint32_t IDESC_QK = ptx::idesc_bf16(128, TOK, 0, 0);
constexpr uint32_t IDESC_PV = ptx::idesc_bf16(128, HC, 0, 1);
static_assert(SMEM_BYTES <= 232448, "shared memory budget");
static_assert((OFF_X % 1024) == 0 && (OFF_P % 1024) == 0 && (OFF_QR % 1024) == 0 &&
                  (OFF_MISC % 1024) == 0 && (STAGE % 1024) == 0, "align");

struct CsMisc {
    uint64_t full[NST], empty[NST];   // KV ring
    uint64_t s_full[2], s_free[2];    // score buffers
    uint64_t x_full[2], x_empty[2];   // peer partial buffers (x_empty counts the peer's readers)
    uint64_t p_ready[2], pv_done[2];  // P buffers / value products
    uint64_t q_ready, q_free, o_free, drain;
    uint32_t tmem_base;
    int32_t abort_flag;
    int32_t cur_b;
    int32_t pad0;
    int64_t cur_O, cur_S, cur_N;
    float xmax[2][2][ROWS];           // half-row maxima, by tile parity and token half
    uint32_t xmax_tag[2][2][ROWS];    // their flags: (tile index / 2) + 1 once written
    float xsum[2][ROWS];              // half-row sums at a segment's end, by token half
    uint32_t xsum_tag[2][ROWS];       // their flags: segment number + 1 once written
};
static_assert(sizeof(CsMisc) <= MISC_BYTES, "misc");

// Byte offset of 16-byte chunk c (0..15) of row r in a partial-score buffer
// ([128 rows x 256 B]); chunks are XOR-swizzled within each 128-byte half so
// that the softmax warps' 16-byte reads spread over all banks.
__device__ __forceinline__ uint32_t xoff(uint32_t r, uint32_t c) {
    return r * 256u + (c & 8u) * 16u + (((c & 7u) ^ (r & 7u)) << 4);
}

// The two threads that hold the halves of one row (in the two softmax warps of
// a lane quadrant) swap a float: each writes its value, then a flag word with
// `tag`, and spins (bounded) until the partner's flag carries the same tag.
// Flags are double-buffered by the caller wherever a slot is reused before
// the partner is known to have read it.
__device__ __forceinline__ bool swap_halves(float *mine, uint32_t *my_tag, const float *theirs,
                                            const uint32_t *their_tag, float v, uint32_t tag,
                                            volatile int32_t *abort_flag, int64_t timeout_ns,
                                            float *out) {
    *mine = v;
    __threadfence_block();
    *reinterpret_cast<volatile uint32_t *>(my_tag) = tag;
    const volatile uint32_t *tt = their_tag;
    if (*tt != tag) {
        const uint64_t t0 = ptx::globaltimer_ns();
        for (uint32_t it = 1; *tt != tag; ++it) {
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
    __threadfence_block();
    *out = *reinterpret_cast<const volatile float *>(theirs);
    return true;
}

// Byte offset of 16-byte chunk c (0..3) of row r in a 64-byte-swizzled block.
__device__ __forceinline__ uint32_t sw64(uint32_t r, uint32_t c) {
    return r * 64u + ((c ^ ((r >> 1) & 3u)) << 4);
}
}  // namespace cs

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(cs::THREADS, 1)
    decode_cs_kernel(const __grid_constant__ CUtensorMap map_ckv, const __grid_constant__ CUtensorMap map_kr,
                     const DecodeArgs args) {
    using namespace cs;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t base = ptx::smem_u32(smem_raw);
    if (base & 1023u) {   // swizzled operands need a 1 KB aligned base; uniform over the cluster
        if (threadIdx.x == 0) record_error(kErrUnsupported);
        return;
    }
    CsMisc *misc = reinterpret_cast<CsMisc *>(smem_raw + OFF_MISC);
    volatile int32_t *abort_flag = &misc->abort_flag;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = ptx::cluster_ctarank();   // channel half
    const uint32_t peer = rank ^ 1u;
    const int64_t part = blockIdx.x >> 1;
    const int64_t P = args.num_parts;
    auto bar = [&](const uint64_t *b) { return ptx::smem_u32(b); };
    auto peer_addr = [&](uint32_t local) { return ptx::mapa(local, peer); };

    // ---------------------------------------------------------------- setup
    if (threadIdx.x == 0) {
        for (int i = 0; i < NST; ++i) {
            ptx::mbar_init(bar(&misc->full[i]), 1);
            ptx::mbar_init(bar(&misc->empty[i]), 1);
        }
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(bar(&misc->s_full[i]), 1);
            ptx::mbar_init(bar(&misc->s_free[i]), 12);    // 8 softmax + 4 sender warps
            ptx::mbar_init(bar(&misc->x_full[i]), 1);     // armed once per tile, + peer bytes
            ptx::mbar_init(bar(&misc->x_empty[i]), 8);    // the peer's softmax warps
            ptx::mbar_init(bar(&misc->p_ready[i]), 8);
            ptx::mbar_init(bar(&misc->pv_done[i]), 1);
        }
        ptx::mbar_init(bar(&misc->q_ready), 4);
        ptx::mbar_init(bar(&misc->q_free), 1);
        ptx::mbar_init(bar(&misc->o_free), 8);
        ptx::mbar_init(bar(&misc->drain), 1);
        misc->abort_flag = 0;
        ptx::fence_mbar_init();
    }
    for (int i = threadIdx.x; i < 2 * 2 * ROWS; i += THREADS) {
        (&misc->xmax_tag[0][0][0])[i] = 0u;
        if (i < 2 * ROWS) (&misc->xsum_tag[0][0])[i] = 0u;
    }
    if (warp == 0) {
        const SeqCursor c = find_sequence(args.seq_lens, args.batch, args.max_pages, args.n_q, TOK,
                                          P, 0);
        const int64_t N = c.total;
        const int64_t ts = (part < c.parts) ? part_start(part, N, c.parts) : N;
        const SeqCursor s = find_sequence(args.seq_lens, args.batch, args.max_pages, args.n_q, TOK,
                                          P, ts);
        if (lane == 0) {
            misc->cur_b = s.b;
            misc->cur_O = s.tile_off;
            misc->cur_S = s.slot_base;
            misc->cur_N = N;
            ptx::prefetch_tensormap(&map_ckv);
            ptx::prefetch_tensormap(&map_kr);
        }
    }
    if (warp == 1) {
        ptx::tmem_alloc<1>(bar(reinterpret_cast<uint64_t *>(&misc->tmem_base)), TMEM_COLS);
        ptx::tmem_relinquish<1>();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::cluster_sync();   // both CTAs' barriers exist before any remote access
    ptx::tc_fence_after();
    const uint32_t tmem = misc->tmem_base;

    SegmentWalker walk;
    walk.seq_lens = args.seq_lens;
    walk.batch = args.batch;
    walk.max_pages = args.max_pages;
    walk.n_q = args.n_q;
    walk.tile_tokens = TOK;
    walk.N = misc->cur_N;
    walk.P = parts_in_use(P, walk.N);
    walk.p = part;
    walk.b = misc->cur_b;
    walk.O = misc->cur_O;
    walk.S = misc->cur_S;
    if (part < walk.P) {
        walk.tile = part_start(part, walk.N, walk.P);
        walk.te = part_start(part + 1, walk.N, walk.P);
    } else {
        walk.tile = walk.te = 0;   // idle partition
    }

    if (warp == 0) {
        // ------------------------------------------------------ TMA producer
        if (ptx::elect_one()) {
            int64_t k = 0;
            bool bad_page = false;
            while (!*abort_flag && walk.next()) {
                const int32_t *trow = args.block_table + static_cast<int64_t>(walk.seg_b) * args.max_pages;
                for (int64_t t = walk.t_begin; t < walk.t_end; ++t, ++k) {
                    const int s = static_cast<int>(k % NST);
                    int32_t page = trow[t];
                    if (page < 0 || page >= args.num_pages) { bad_page = true; page = 0; }
                    if (k >= NST && !wait_bounded<false>(bar(&misc->empty[s]), ((k / NST) - 1) & 1,
                                                         abort_flag, args.timeout_ns))
                        break;
                    const uint32_t fb = bar(&misc->full[s]);
                    ptx::mbar_arrive_expect_tx(fb, STAGE);
                    const uint32_t st = base + OFF_KV + s * STAGE;
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        ptx::tma_load_3d(st + u * BLK, &map_ckv, fb, 64 * (4 * static_cast<int>(rank) + u),
                                         0, page);
                    ptx::tma_load_3d(st + 4 * BLK, &map_kr, fb, HR * static_cast<int>(rank), 0, page);
                }
            }
            if (bad_page) record_error(kErrDeviceBounds);
            for (int64_t kk = (k >= NST ? k - NST : 0); kk < k; ++kk)
                wait_bounded<false>(bar(&misc->full[kk % NST]), (kk / NST) & 1, abort_flag,
                                    args.timeout_ns);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------ MMA issuer
        // Two cursors: QK^T of tile kq and P.V of tile kp (kp < kq <= kp + 2,
        // two score buffers); whichever is ready is issued.
        if (ptx::elect_one()) {
            SegmentWalker wq = walk, wp = walk;
            bool q_has = wq.next(), p_has = wp.next();
            int64_t tq = q_has ? wq.t_begin : 0, tp = p_has ? wp.t_begin : 0;
            int64_t kq = 0, kp = 0, gq = 0, gp = 0;
            bool q_ready_seen = false, o_free_seen = false;
            uint64_t idle_since = ptx::globaltimer_ns();
            uint32_t spins = 0;
            while ((q_has || p_has) && !*abort_flag) {
                bool progressed = false;
                if (q_has && kq < kp + 2) {
                    if (!q_ready_seen) q_ready_seen = ptx::mbar_test_wait(bar(&misc->q_ready), gq & 1);
                    const int s = static_cast<int>(kq % NST);
                    const int b = static_cast<int>(kq & 1);
                    if (q_ready_seen &&
                        ptx::mbar_test_wait(bar(&misc->full[s]), (kq / NST) & 1) &&
                        (kq < 2 || ptx::mbar_test_wait(bar(&misc->s_free[b]), ((kq >> 1) - 1) & 1))) {
                        ptx::tc_fence_after();
                        const uint32_t st = base + OFF_KV + s * STAGE;
                        const uint32_t d = tmem + TMEM_S + 64 * b;
#pragma unroll
                        for (int j = 0; j < HC / 16; ++j) {   // latent: A (Q) from tensor memory
                            const uint64_t bd = ptx::smem_desc(st + (j >> 2) * BLK + (j & 3) * 32, 16,
                                                               1024, ptx::kSwizzle128B);
                            ptx::mma_bf16_ts<1>(d, tmem + TMEM_Q + 8 * j, bd, IDESC_QK, j ? 1u : 0u);
                        }
#pragma unroll
                        for (int j = 0; j < HR / 16; ++j) {   // RoPE: both operands from shared memory
                            const uint64_t ad = ptx::smem_desc(base + OFF_QR + 32 * j, 16, 512,
                                                               ptx::kSwizzle64B);
                            const uint64_t bd = ptx::smem_desc(st + 4 * BLK + 32 * j, 16, 512,
                                                               ptx::kSwizzle64B);
                            ptx::mma_bf16_ss<1>(d, ad, bd, IDESC_QK, 1u);
                        }
                        ptx::mma_commit(bar(&misc->s_full[b]));
                        ++kq;
                        if (++tq == wq.t_end) {
                            ptx::mma_commit(bar(&misc->q_free));   // Q may be replaced
                            q_has = wq.next();
                            ++gq;
                            q_ready_seen = false;
                            if (q_has) tq = wq.t_begin;
                        }
                        progressed = true;
                    }
                }
                if (p_has && kp < kq) {
                    const bool first = (tp == wp.t_begin);
                    if (first && gp > 0 && !o_free_seen)
                        o_free_seen = ptx::mbar_test_wait(bar(&misc->o_free), (gp - 1) & 1);
                    const int b = static_cast<int>(kp & 1);
                    const int s = static_cast<int>(kp % NST);
                    if ((!first || gp == 0 || o_free_seen) &&
                        ptx::mbar_test_wait(bar(&misc->p_ready[b]), (kp >> 1) & 1)) {
                        ptx::tc_fence_after();
                        const uint32_t st = base + OFF_KV + s * STAGE;
#pragma unroll
                        for (int kk = 0; kk < TOK / 16; ++kk) {
                            const uint64_t ad = ptx::smem_desc(base + OFF_P + b * PBUF + 32 * kk, 16,
                                                               1024, ptx::kSwizzle128B);
                            const uint64_t bd = ptx::smem_desc(st + 2048 * kk, BLK, 1024,
                                                               ptx::kSwizzle128B);
                            ptx::mma_bf16_ss<1>(tmem + TMEM_O, ad, bd, IDESC_PV,
                                                (first && kk == 0) ? 0u : 1u);
                        }
                        ptx::mma_commit(bar(&misc->pv_done[b]));
                        ptx::mma_commit(bar(&misc->empty[s]));   // QK^T and P.V of the stage done
                        ++kp;
                        if (++tp == wp.t_end) {
                            p_has = wp.next();
                            ++gp;
                            o_free_seen = false;
                            if (p_has) tp = wp.t_begin;
                        }
                        progressed = true;
                    }
                }
                if (progressed) {
                    spins = 0;
                } else if ((++spins & 63u) == 0u) {
                    const uint64_t now = ptx::globaltimer_ns();
                    if (spins == 64u) idle_since = now;
                    else if (static_cast<int64_t>(now - idle_since) > args.timeout_ns) {
                        record_error(kErrTimeout);
                        *abort_flag = 1;
                    }
                }
            }
            ptx::mma_commit(bar(&misc->drain));
            wait_bounded<false>(bar(&misc->drain), 0, abort_flag, args.timeout_ns);
        }
    } else if (warp >= SND0) {
        // ------------------------------------------------------ senders + Q loads
        const int q4 = warp & 3;
        const int row = q4 * 32 + lane;                 // TMEM lane = query row
        const bool real_row = row < args.rows;
        const uint32_t lane_base = static_cast<uint32_t>(q4 * 32) << 16;
        auto load_q = [&](int32_t b) {
            // latent channels of this half -> tensor memory (bf16 pairs per column),
            // RoPE channels of this half -> shared memory (64-byte swizzle)
            const __nv_bfloat16 *qrow = args.q + (static_cast<int64_t>(b) * args.rows +
                                                  (real_row ? row : 0)) * D;
#pragma unroll 1
            for (int h = 0; h < 2; ++h) {
                uint4 v[16];
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    v[i] = real_row ? ld_global_nc_v4(qrow + HC * rank + 128 * h + 8 * i)
                                    : make_uint4(0, 0, 0, 0);
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    uint32_t w[32];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        w[4 * i] = v[8 * c + i].x;
                        w[4 * i + 1] = v[8 * c + i].y;
                        w[4 * i + 2] = v[8 * c + i].z;
                        w[4 * i + 3] = v[8 * c + i].w;
                    }
                    ptx::tmem_st32(tmem + lane_base + TMEM_Q + 64 * h + 32 * c, w);
                }
            }
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint4 v = real_row ? ld_global_nc_v4(qrow + DC + HR * rank + 8 * c) : make_uint4(0, 0, 0, 0);
                st_shared_v4(base + OFF_QR + sw64(row, c), v.x, v.y, v.z, v.w);
            }
            ptx::tmem_wait_st();
            ptx::fence_proxy_async_smem();
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(bar(&misc->q_ready));
        };
        auto prefetch_q = [&](int32_t b) {   // the next segment's Q rows into L2
            if (!real_row) return;
            const __nv_bfloat16 *qrow = args.q + (static_cast<int64_t>(b) * args.rows + row) * D;
#pragma unroll
            for (int i = 0; i < 4; ++i) ptx::prefetch_l2(qrow + HC * rank + 64 * i);
            ptx::prefetch_l2(qrow + DC + HR * rank);
        };
        const uint32_t xbase_peer = peer_addr(base + OFF_X);
        int64_t k = 0, g = 0;
        bool have = walk.next();
        if (have) load_q(walk.seg_b);
        while (have && !*abort_flag) {
            {
                SegmentWalker nx = walk;
                if (nx.next()) prefetch_q(nx.seg_b);
            }
            bool ok = true;
            for (int64_t t = walk.t_begin; t < walk.t_end; ++t, ++k) {
                const int b = static_cast<int>(k & 1);
                if (!wait_bounded<false>(bar(&misc->s_full[b]), (k >> 1) & 1, abort_flag,
                                         args.timeout_ns)) { ok = false; break; }
                ptx::tc_fence_after();
                uint32_t s0[32], s1[32];
                ptx::tmem_ld32_pair(tmem + lane_base + TMEM_S + 64 * b, s0, s1);
                ptx::tmem_wait_ld();
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(bar(&misc->s_free[b]));
                // the peer's buffer b is free once its readers of tile k - 2 are done
                if (k >= 2 && !wait_bounded(bar(&misc->x_empty[b]), ((k >> 1) - 1) & 1, abort_flag,
                                            args.timeout_ns)) { ok = false; break; }
                const uint32_t xb = xbase_peer + b * XBUF;
                const uint32_t xbar = peer_addr(bar(&misc->x_full[b]));
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    ptx::st_async_v4(xb + xoff(row, c), s0[4 * c], s0[4 * c + 1], s0[4 * c + 2],
                                     s0[4 * c + 3], xbar);
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    ptx::st_async_v4(xb + xoff(row, 8 + c), s1[4 * c], s1[4 * c + 1], s1[4 * c + 2],
                                     s1[4 * c + 3], xbar);
            }
            if (!ok) break;
            have = walk.next();
            if (have) {
                // Q of the next segment once the last QK^T of this one is done
                if (!wait_bounded<false>(bar(&misc->q_free), g & 1, abort_flag, args.timeout_ns)) break;
                ptx::tc_fence_after();
                load_q(walk.seg_b);
            }
            ++g;
        }
    } else {
        // ------------------------------------------------------ softmax / epilogue
        const int gi = warp - SMX0;                    // 0..7
        const int q4 = warp & 3;                       // TMEM lane quadrant
        const int jh = gi >> 2;                        // token half of the tile (and column half of O)
        const int row = q4 * 32 + lane;                // TMEM lane = query row
        const bool real_row = row < args.rows;
        const int qi = real_row ? row / args.heads : 0;
        const uint32_t lane_addr = static_cast<uint32_t>(q4 * 32) << 16;
        const int st_tid = threadIdx.x - SMX0 * 32;    // 0..255
        const uint32_t xempty_peer0 = peer_addr(bar(&misc->x_empty[0]));
        const uint32_t xempty_peer1 = peer_addr(bar(&misc->x_empty[1]));

        int64_t k = 0, seg_no = 0;
        while (!*abort_flag && walk.next()) {
            const int32_t L = walk.L;
            const int64_t slot = walk.slot;
            const int64_t k0 = k;
            const int32_t vis = real_row ? (L - args.n_q + qi + 1) : 0;
            float m_run = -INFINITY;      // running max (raw score units), same in both threads of a row
            float l_half = 0.f;           // this thread's share of the row sum
            bool ok = true;
            for (int64_t t = walk.t_begin; t < walk.t_end; ++t, ++k) {
                const int b = static_cast<int>(k & 1);
                if (!wait_bounded<false>(bar(&misc->s_full[b]), (k >> 1) & 1, abort_flag,
                                         args.timeout_ns)) { ok = false; break; }
                ptx::tc_fence_after();
                uint32_t sr[32];
                ptx::tmem_ld32(tmem + lane_addr + TMEM_S + 64 * b + 32 * jh, sr);
                if (gi == 0 && lane == 0)   // arm this tile's receive buffer: the peer's bytes
                    ptx::mbar_arrive_expect_tx(bar(&misc->x_full[b]), XBUF);
                ptx::tmem_wait_ld();
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(bar(&misc->s_free[b]));   // score buffer read
                if (!wait_bounded(bar(&misc->x_full[b]), (k >> 1) & 1, abort_flag, args.timeout_ns)) {
                    ok = false;
                    break;
                }
                const uint32_t xb = base + OFF_X + b * XBUF;
                float v[32];
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    uint4 x;
                    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                                 : "=r"(x.x), "=r"(x.y), "=r"(x.z), "=r"(x.w)
                                 : "r"(xb + xoff(row, 8 * jh + c)));
                    v[4 * c] = __uint_as_float(sr[4 * c]) + __uint_as_float(x.x);
                    v[4 * c + 1] = __uint_as_float(sr[4 * c + 1]) + __uint_as_float(x.y);
                    v[4 * c + 2] = __uint_as_float(sr[4 * c + 2]) + __uint_as_float(x.z);
                    v[4 * c + 3] = __uint_as_float(sr[4 * c + 3]) + __uint_as_float(x.w);
                }
                __syncwarp();
                if (lane == 0)   // the peer may refill buffer b
                    ptx::mbar_arrive_cluster_release(b ? xempty_peer1 : xempty_peer0);

                const int32_t tok0 = static_cast<int32_t>(t) * TOK + jh * 32;
                float mx = -INFINITY;
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    v[j] = (tok0 + j < vis) ? v[j] : -INFINITY;
                    mx = fmaxf(mx, v[j]);
                }
                {   // the two halves of the row meet
                    float other;
                    const int pk = static_cast<int>(k & 1);
                    if (!swap_halves(&misc->xmax[pk][jh][row], &misc->xmax_tag[pk][jh][row],
                                     &misc->xmax[pk][jh ^ 1][row], &misc->xmax_tag[pk][jh ^ 1][row], mx,
                                     static_cast<uint32_t>(k >> 1) + 1u, abort_flag, args.timeout_ns,
                                     &other)) { ok = false; break; }
                    mx = fmaxf(mx, other);
                }
                float alpha = 1.f;
                if (mx > -INFINITY && (m_run == -INFINITY ||
                                       (mx - m_run) * args.scale_log2 > kRescaleThreshold)) {
                    alpha = (m_run == -INFINITY) ? 0.f : exp2f((m_run - mx) * args.scale_log2);
                    m_run = mx;
                }
                const float mb = (m_run == -INFINITY) ? 0.f : m_run * args.scale_log2;
                float ps[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    v[j] = exp2f(fmaf(v[j], args.scale_log2, -mb));   // -inf -> 0
                    ps[j & 3] += v[j];
                }
                l_half = fmaf(l_half, alpha, (ps[0] + ps[1]) + (ps[2] + ps[3]));

                // rescale this row's accumulated O (this thread: 128 of the 256 columns)
                const bool need = (k > k0) && (alpha != 1.f);
                const bool any_need = __any_sync(0xffffffffu, need);
                if (any_need) {
                    const int64_t kp = k - 1;
                    if (!wait_bounded<false>(bar(&misc->pv_done[kp & 1]), (kp >> 1) & 1, abort_flag,
                                             args.timeout_ns)) { ok = false; break; }
                    ptx::tc_fence_after();
#pragma unroll 1
                    for (int c = 0; c < 4; ++c) {
                        uint32_t o[32];
                        const uint32_t ta = tmem + lane_addr + TMEM_O + 128 * jh + 32 * c;
                        ptx::tmem_ld32(ta, o);
                        ptx::tmem_wait_ld();
#pragma unroll
                        for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha);
                        ptx::tmem_st32(ta, o);
                    }
                    ptx::tmem_wait_st();
                }
                // P buffer b is free once the value product of tile k - 2 is done
                if (k >= 2 && !wait_bounded<false>(bar(&misc->pv_done[b]), ((k >> 1) - 1) & 1,
                                                   abort_flag, args.timeout_ns)) { ok = false; break; }
                const uint32_t pb = base + OFF_P + b * PBUF;
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    st_shared_v4(pb + sw128(row, 4 * jh + c), pack_bf16x2(v[8 * c + 0], v[8 * c + 1]),
                                 pack_bf16x2(v[8 * c + 2], v[8 * c + 3]),
                                 pack_bf16x2(v[8 * c + 4], v[8 * c + 5]),
                                 pack_bf16x2(v[8 * c + 6], v[8 * c + 7]));
                // Last tile of the sequence: the page's rows past its end were loaded
                // with the page and may hold any bits (an unwritten or recycled slot).
                // Their P is 0, but 0 * NaN = NaN in the value product, so they are
                // cleared; QK^T of this tile has read the stage (s_full) and P.V
                // waits for p_ready.
                const int32_t valid = L - static_cast<int32_t>(t) * TOK;
                if (valid < TOK) {
                    const uint32_t st = base + OFF_KV + static_cast<uint32_t>(k % NST) * STAGE;
                    const int n16 = (TOK - valid) * 8;   // 16-byte chunks per channel block
                    for (int idx = st_tid; idx < 4 * n16; idx += 256) {
                        const int u = idx / n16, rem = idx - u * n16;
                        st_shared_v4(st + u * BLK + (valid + (rem >> 3)) * 128 + (rem & 7) * 16, 0u,
                                     0u, 0u, 0u);
                    }
                }
                ptx::fence_proxy_async_smem();
                if (any_need) ptx::tc_fence_before();   // order the O rescale stores
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(bar(&misc->p_ready[b]));
            }
            if (!ok) break;

            // epilogue of this segment: O_h / l for this CTA's channels
            const int64_t kl = k - 1;
            if (!wait_bounded<false>(bar(&misc->pv_done[kl & 1]), (kl >> 1) & 1, abort_flag,
                                     args.timeout_ns))
                break;
            ptx::tc_fence_after();
            // both halves added in the same order by both threads of the row
            float l_other;
            if (!swap_halves(&misc->xsum[jh][row], &misc->xsum_tag[jh][row], &misc->xsum[jh ^ 1][row],
                             &misc->xsum_tag[jh ^ 1][row], l_half, static_cast<uint32_t>(seg_no) + 1u,
                             abort_flag, args.timeout_ns, &l_other))
                break;
            ++seg_no;
            const float l_row = jh ? (l_other + l_half) : (l_half + l_other);
            const float inv = (l_row > 0.f) ? 1.f / l_row : 0.f;
            float *dst = args.o_part + (slot * args.rows + row) * DC + HC * rank + 128 * jh;
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
                uint32_t o[32];
                ptx::tmem_ld32(tmem + lane_addr + TMEM_O + 128 * jh + 32 * c, o);
                ptx::tmem_wait_ld();
                if (real_row) {
                    float4 *d4 = reinterpret_cast<float4 *>(dst + 32 * c);
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        d4[j] = make_float4(__uint_as_float(o[4 * j]) * inv,
                                            __uint_as_float(o[4 * j + 1]) * inv,
                                            __uint_as_float(o[4 * j + 2]) * inv,
                                            __uint_as_float(o[4 * j + 3]) * inv);
                }
            }
            if (real_row && rank == 0 && jh == 0)
                args.lse_part[slot * args.rows + row] =
                    (l_row > 0.f) ? m_run * args.scale + logf(l_row) : -INFINITY;
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(bar(&misc->o_free));
        }
    }

    // ---------------------------------------------------------------- teardown
    ptx::tc_fence_before();
    __syncthreads();
    ptx::cluster_sync();   // no remote store or arrive targets a CTA that has left
    ptx::tc_fence_after();
    if (warp == 1) ptx::tmem_dealloc<1>(tmem, TMEM_COLS);
}

}  // namespace mla
