// Split-KV MLA decode in latent space on sm_100a tensor cores.
//
// What one partition computes (absorbed score and value steps; "MLA operator
// design" page §4 path B, "MHA2MLA" page §2.1):
//   S = Q [c_KV | k_R]^T                      (all heads share one latent KV)
//   online softmax over the partition's tokens (fp32, exp2 domain)
//   O = P c_KV                                (value product stays in latent space)
//   partial = O / l,  lse = m * scale + ln l
//
// Two kernels share the pipeline shape: TMA producer warps stream KV pages
// into shared-memory rings, one thread of warp 1 issues tcgen05 MMAs into
// tensor memory, and warps 2..5 run the softmax, rescale O when the running
// maximum grows by more than 2^8, write P, and write the partials.
//
//  * decode_pair_kernel (d_c 512, d_R 64, page = tile = 64 tokens): a CTA pair
//    on two SMs. The fp32 accumulator O[128 rows x 512] is exactly one SM's
//    256 KB of tensor memory, so the pair splits it: cta_group::2 MMAs with
//    M = 128 give each SM the O rows of its 64 query rows. QK^T splits the
//    tile's 64 tokens (32 per SM); P.V splits the 512 latent columns (256 per
//    SM, as two N = 256 MMAs). No MMA work is duplicated. Six of Q's nine
//    64-channel blocks are the QK^T A operand straight from tensor memory,
//    which leaves shared memory for a three-slot QK^T ring.
//  * decode_single_kernel (d_c 64, d_R 8, tile = 128 tokens = 2 pages): one
//    CTA, cta_group::1, M = 128 rows; the 8-wide RoPE key is padded to the
//    16-wide MMA K step with a zero core-matrix column in shared memory.
//
// Every wait is bounded (see wait_bounded); data errors set the device error
// word. The kernels never read block-table entries past a sequence's last
// page.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda.h>

#include "common.cuh"

namespace mla {

struct DecodeArgs {
    const __nv_bfloat16 *q;      // [B, R, D]
    const int32_t *block_table;  // [B, max_pages]
    const int32_t *seq_lens;     // [B]
    const float *kv_scales;      // E4M3 cache: per-token scales [pages, 64] (else unused)
    float *o_part;               // [slots, R, d_c]
    float *lse_part;             // [slots, R]
    int64_t timeout_ns;
    int32_t max_pages;
    int32_t batch;
    int32_t num_pages;
    int32_t num_parts;
    int32_t n_q;
    int32_t heads;
    int32_t rows;                // R = n_q * heads (<= 128)
    float scale;                 // softmax scale
    float scale_log2;            // scale * log2(e)
};

constexpr int kDecodeThreads = 192;          // single kernel: 6 warps
constexpr int kPairThreads = 352;            // pair kernel: 11 warps (6 = P.V-slot producer, 7..10 segment warps)
constexpr int kSegWarp0 = 7;                 // pair kernel: first of the four segment warps
constexpr int kPairThreadsFp8 = 480;         // E4M3 pair kernel: + 4 dequantising warps (11..14)
constexpr int kDqWarp0 = 11;
constexpr int kSoftmaxWarp0 = 2;             // warps 2..5
constexpr float kRescaleThreshold = 8.0f;    // log2 units: rescale O when max grows > 2^8

// ------------------------------------------------------------------ helpers

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
                 "r"(d)
                 : "memory");
}

__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr)
                 : "memory");
    return v;
}

__device__ __forceinline__ uint4 ld_global_nc_v4(const void *p) {
    uint4 v;
    asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// Maximum of N values as eight interleaved chains and a tree (short
// dependency depth; max is exact in any order).
template <int N>
__device__ __forceinline__ float max_of(const float (&v)[N]) {
    static_assert(N % 8 == 0, "N");
    float m[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) m[i] = v[i];
#pragma unroll
    for (int j = 8; j < N; ++j) m[j & 7] = fmaxf(m[j & 7], v[j]);
    return fmaxf(fmaxf(fmaxf(m[0], m[1]), fmaxf(m[2], m[3])), fmaxf(fmaxf(m[4], m[5]), fmaxf(m[6], m[7])));
}

// Byte offset of 16-byte chunk `chunk` (0..7) of row `row` inside a
// 128-byte-swizzled K-major block whose rows are 128 bytes apart.
__device__ __forceinline__ uint32_t sw128(uint32_t row, uint32_t chunk) {
    return row * 128u + ((chunk ^ (row & 7u)) << 4);
}

// Iterates the (sequence, tile range) segments of one partition: the tiles
// whose plan cost position falls in [tile, te). Every thread that walks it gets
// the same sequence of segments.
struct SegmentWalker {
    const int32_t *seq_lens;
    int32_t batch, max_pages, n_q, tile_tokens;
    int64_t N, P, p, te;   // N: plan cost C; te: end of this partition's cost range
    // current state
    int32_t b;
    int64_t O, S, tile;    // O: cost offset C_b of sequence b; tile: cost position reached
    // current segment
    int32_t seg_b, L;
    int64_t t_begin, t_end, slot;
    bool primed = false;   // the current segment was found ahead: next() hands it out

    __device__ bool next() {
        if (primed) {
            primed = false;
            return true;
        }
        while (tile < te && b < batch) {
            bool bad = false;
            const int32_t Lb = clamp_len(seq_lens[b], max_pages, n_q, &bad);
            const int64_t n = tiles_of_len(Lb, tile_tokens);
            if (n == 0) { ++b; continue; }
            if (O >= te) return false;   // the next sequence starts past this partition
            const int64_t pf = part_of_tile(O, N, P);
            seg_b = b;
            L = Lb;
            t_begin = (tile > O) ? tile - O : 0;
            t_end = (te - O < n) ? (te - O) : n;
            slot = S + (p - pf);
            tile = O + t_end;
            const int64_t pl = part_of_tile(O + n - 1, N, P);
            S += pl - pf + 1;
            O += n + switch_cost(tile_tokens);
            ++b;
            return true;
        }
        return false;
    }
};

// ===========================================================================
// CTA-pair kernel: d_c = 512, d_R = 64
// ===========================================================================
namespace pair {
constexpr int DC = 512, DR = 64, D = DC + DR;
constexpr int NB = D / 64;                    // 9 K-blocks of 64 channels
constexpr int ROWS_CTA = 64;                  // query rows per SM
constexpr int TOK = 64;                       // tokens per tile (one page)
constexpr int OWN = 32;                       // tokens per SM in QK^T
constexpr int QT = 5;                         // Q channel blocks 0..4 live in tensor memory
constexpr int NSB = 3;                        // score buffers in tensor memory
constexpr uint32_t Q_BYTES = (NB - QT) * ROWS_CTA * 128;    // 32768: Q blocks 5..8
constexpr uint32_t STAGE_QK = NB * OWN * 128;               // 36864: own 32 tokens x 9 blocks
constexpr uint32_t STAGE_PV = 4 * TOK * 128;                // 32768: 64 tokens x this SM's 4 blocks
constexpr int QK_STAGES = 3;                                // QK^T ring depth
constexpr int PV_STAGES = 2;                                // P.V ring depth
constexpr uint32_t P_BYTES = ROWS_CTA * 128;                // 64 rows x 64 tokens bf16
constexpr uint32_t OFF_Q = 0;
constexpr uint32_t OFF_QK = OFF_Q + Q_BYTES;                // QK^T ring
constexpr uint32_t OFF_PV = OFF_QK + QK_STAGES * STAGE_QK;  // P.V ring
constexpr uint32_t OFF_P = OFF_PV + PV_STAGES * STAGE_PV;
constexpr uint32_t OFF_MISC = OFF_P + 2 * P_BYTES;          // 217088
constexpr uint32_t MISC_BYTES = 3072;
constexpr uint32_t OFF_EPI = OFF_MISC + MISC_BYTES;         // partial-store staging, 1 KB per segment warp
constexpr uint32_t EPI_BYTES = 4 * 32 * 32;
constexpr uint32_t SMEM_BYTES = OFF_EPI + EPI_BYTES;     // dynamic smem base is 1 KB aligned
// The first segment's Q blocks 0..QT-1 land here by TMA before they are copied to
// tensor memory: P.V slot 1 and P buffer 0, which nothing uses until Q is ready
// (the P.V producer waits for q_stage_free before its first copy into slot 1).
constexpr uint32_t OFF_QSTAGE = OFF_PV + STAGE_PV;
// The first segment's first FIRST_PAGES page numbers, read with the plan, wait in
// the partial-store staging tile: the producers read them at once after setup,
// and the segment warps first write there at that segment's end.
constexpr int FIRST_PAGES = 4;
constexpr uint32_t OFF_FIRST_PAGES = OFF_EPI;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TMEM_O = 0;                 // two 128-column accumulators (c = 0, 1)
constexpr uint32_t TMEM_S = 256;               // three 32-column score buffers
constexpr uint32_t TMEM_Q = TMEM_S + NSB * 32; // Q blocks 0..4: 32 columns each (two bf16 per column)
constexpr uint32_t IDESC_QK = ptx::idesc_bf16(128, TOK, 0, 0);
constexpr uint32_t IDESC_PV = ptx::idesc_bf16(128, 256, 0, 1);
// E4M3 cache: a slot's c_KV codes land in bytes [CODE_OFF, CODE_OFF + CODE_BYTES)
// of the slot and are widened in place to the bf16 operand above.
constexpr uint32_t CODE_OFF = 16384;
constexpr uint32_t CODE_BYTES = 16384;         // QK^T: 32 tokens x 512; P.V: 64 tokens x 256
constexpr uint32_t SC_BYTES = 4 * 32 * 4;      // four copies of 32 tokens' scales per slot
static_assert(SMEM_BYTES <= 232448, "shared memory budget");
static_assert(TMEM_Q + QT * 32 <= TMEM_COLS, "tensor memory budget");
static_assert(PV_STAGES == 2 && OFF_QSTAGE + QT * ROWS_CTA * 128 <= OFF_P + P_BYTES, "Q staging");
static_assert((OFF_QK % 1024) == 0 && (OFF_PV % 1024) == 0 && (OFF_P % 1024) == 0 &&
                  (OFF_MISC % 1024) == 0, "align");
}  // namespace pair

// misc-region layout (both kernels)
struct Misc {
    uint64_t full[2], empty[2], s_full[pair::NSB], s_free[2], p_ready[2], pv_done[2], q_ready, o_free;
    uint64_t drain;                   // MMA drain before tensor memory is freed
    uint64_t qk_full[pair::QK_STAGES], qk_empty[pair::QK_STAGES];   // the pair kernel's two rings
    uint64_t pv_full[pair::PV_STAGES], pv_empty[pair::PV_STAGES];
    uint64_t pv_landed[pair::PV_STAGES];   // pair kernel: a P.V slot has landed (both CTAs)
    uint32_t tmem_base;
    int32_t abort_flag;
    int32_t cur_b;
    int32_t pad0;
    int64_t cur_O, cur_S, cur_N, cur_P;   // plan: cost offset, slot base, total cost, partitions
    uint32_t xtag[2][128];            // pair kernel: tagged half-row maxima, by tile parity
    uint32_t xltag[128];              // pair kernel: tagged half-row sums, by segment
    uint64_t q_free;                  // pair kernel: the last QK^T of a segment is done (Q may be replaced)
    uint64_t seg_done;                // pair kernel: a segment's row sums and maxima are published
    float seg_l[2][64], seg_m[2][64]; // pair kernel: those sums and maxima, by segment parity
    uint64_t code_qk[pair::QK_STAGES], code_pv[pair::PV_STAGES];   // E4M3 pair kernel: codes landed
    uint64_t kv_full[8], kv_empty[8];   // single kernel: its KV ring
    // the partition's first segment, found before the dependency wait (the
    // walker's state after its first next(); first_b < 0: none)
    int64_t first_tile, first_slot;
    int32_t first_b, first_L, first_t_begin, first_t_end;
    uint64_t q_tma;                   // pair kernel: the first segment's Q has landed
    uint64_t q_stage_free;            // pair kernel: its staged blocks are in tensor memory
};
static_assert(sizeof(Misc) <= pair::MISC_BYTES, "misc");

// Tile-by-tile walk over a partition's segments.
struct TileCursor {
    SegmentWalker w;
    bool have;
    int64_t t;   // tile index within sequence w.seg_b
    __device__ void start() {
        have = w.next();
        t = have ? w.t_begin : 0;
    }
    __device__ void advance() {
        if (++t >= w.t_end) {
            have = w.next();
            if (have) t = w.t_begin;
        }
    }
};

// E4M3 pair kernel: one warp widens its share of a ring slot's codes in place.
// The codes sit at slot + CODE_OFF as NBOX boxes of [rows x 128 codes] (box v:
// 128 consecutive channels of the slot's channel range, rows = blk / 128); the
// bf16 operand is block j = 2v + e ([rows x 64 channels], 128-byte swizzled) at
// slot + j * blk. The warp owns 8 NPAIR slot rows from wrow0 on; lane
// (c = lane & 7, q = lane >> 3) converts 16-code chunk c of rows
// row(pr, h) = wrow0 + 2 (q + 4 pr) + ((c / 4) ^ h) & 1 of every box, for its
// NPAIR row pairs pr. A quarter-warp's two rows alternate with c, so its reads
// cover 128 contiguous bytes and its stores fall in distinct banks. The units
// (box, pr) go in order, two per step: a step's codes are read by every lane
// before the warp syncs and any lane writes the step's outputs. An output row
// overlaps only codes of the same row, of this box or an earlier one, so every
// code is read before it is overwritten; the next step's codes (never written
// by this step) are loaded before this step's stores, which hides the load
// latency. Rows at or past rlim (tokens past the sequence end) are written as
// zeros. The loop stays rolled: one step of straight-line code.
template <int NBOX, int NPAIR>
__device__ __forceinline__ void dequant_slot(uint32_t slot, uint32_t blk, int wrow0, int lane, int32_t rlim,
                                             const float (&sc)[2 * NPAIR]) {
    constexpr int NST = NBOX * NPAIR / 2;   // steps of two units
    static_assert(NPAIR <= 2, "a step's scales are fixed");
    const int c = lane & 7, q = lane >> 3;
    const uint32_t codes = slot + pair::CODE_OFF + c * 16;
    auto row = [&](int pr, int h) { return wrow0 + 2 * (q + 4 * pr) + (((c >> 2) ^ h) & 1); };
    // row(pr, h) mod 8 does not depend on pr, so neither do the swizzled chunk
    // offsets of the two 16-byte outputs: (2 (c mod 4) + x) ^ (row mod 8), x = 0, 1
    uint32_t xo[2][2];
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int x = 0; x < 2; ++x) xo[h][x] = static_cast<uint32_t>(((2 * (c & 3) + x) ^ (row(0, h) & 7)) << 4);
    // unit un: box un / NPAIR, pair un % NPAIR (compile-time within a step but for the box)
    auto load = [&](int st, uint4 (&v)[4]) {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int un = 2 * st + (u >> 1);
            v[u] = ld_shared_v4(codes + (un / NPAIR) * blk + row(un % NPAIR, u & 1) * 128);
        }
    };
    uint4 v[4];
    load(0, v);
#pragma unroll 1
    for (int st = 0; st < NST; ++st) {
        __syncwarp();   // every lane has read this step's codes
        uint4 o[8];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            // scale of row(pr, h): entry 2 pr + h; within a step pr = (2 st + u / 2) % NPAIR
            // is u / 2 for NPAIR 2 and 0 for NPAIR 1
            const float s = sc[(NPAIR == 2 ? 2 * (u >> 1) : 0) + (u & 1)];
            const uint2 d0 = dequant4_e4m3(v[u].x, s);
            const uint2 d1 = dequant4_e4m3(v[u].y, s);
            const uint2 d2 = dequant4_e4m3(v[u].z, s);
            const uint2 d3 = dequant4_e4m3(v[u].w, s);
            o[2 * u] = make_uint4(d0.x, d0.y, d1.x, d1.y);
            o[2 * u + 1] = make_uint4(d2.x, d2.y, d3.x, d3.y);
        }
        uint4 nv[4];
        if (st + 1 < NST) load(st + 1, nv);   // the next step's codes: rows or boxes this step does not write
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int un = 2 * st + (u >> 1);
            const int r = row(un % NPAIR, u & 1);
            uint4 lo = o[2 * u], hi = o[2 * u + 1];
            if (r >= rlim) lo = hi = make_uint4(0u, 0u, 0u, 0u);
            // sw128(r, chunk) = r * 128 + xo
            const uint32_t rb = slot + (2 * (un / NPAIR) + (c >> 2)) * blk + static_cast<uint32_t>(r) * 128u;
            st_shared_v4(rb + xo[u & 1][0], lo.x, lo.y, lo.z, lo.w);
            st_shared_v4(rb + xo[u & 1][1], hi.x, hi.y, hi.z, hi.w);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) v[u] = nv[u];
    }
}

// E4M3 pair kernel: one dequantising warp's share of one slot: wait until the
// slot's codes and scales have landed, widen them, report the slot full on the
// leader's barrier. The scales (32 consecutive tokens, from slot row sc_row0
// on) arrive by TMA in the warp's own last row of block NBOX - 1, which the
// warp itself overwrites in its first step, after reading them.
template <int NBOX, int NPAIR>
__device__ __forceinline__ bool dequant_tile(const TileCursor &cur, int64_t k, const DecodeArgs &args,
                                             uint32_t ring, uint32_t stage, uint32_t blk, int nst,
                                             uint64_t *codeb, uint64_t *fullb, int wrow0, int sc_row0,
                                             int tok_off, uint32_t rank, int lane,
                                             volatile int32_t *abort_flag) {
    const int c = lane & 7, q = lane >> 3;
    const int s = static_cast<int>(k % nst);
    if (!wait_bounded<false>(ptx::smem_u32(&codeb[s]), (k / nst) & 1, abort_flag, args.timeout_ns))
        return false;
    const uint32_t slot = ring + s * stage;
    const uint32_t sc_off = (NBOX - 1) * blk + (wrow0 + 8 * NPAIR - 1) * 128;
    float sc[2 * NPAIR];
#pragma unroll
    for (int i = 0; i < 2 * NPAIR; ++i) {
        const int r = wrow0 + 2 * (q + 4 * (i >> 1)) + (((c >> 2) ^ i) & 1);
        asm volatile("ld.shared.f32 %0, [%1];" : "=f"(sc[i]) : "r"(slot + sc_off + 4 * (r - sc_row0)) : "memory");
    }
    __syncwarp();   // the scale row is overwritten below
    const int32_t rlim = cur.w.L - static_cast<int32_t>(cur.t) * pair::TOK - tok_off;
    dequant_slot<NBOX, NPAIR>(slot, blk, wrow0, lane, rlim, sc);
    ptx::fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
        const uint32_t fb = ptx::smem_u32(&fullb[s]);
        if (rank == 0) ptx::mbar_arrive(fb);
        else ptx::mbar_arrive_cluster(ptx::mapa(fb, 0));
    }
    return true;
}

template <bool kFp8>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kFp8 ? kPairThreadsFp8 : kPairThreads, 1)
    decode_pair_kernel(const __grid_constant__ CUtensorMap map_ckv32,
                       const __grid_constant__ CUtensorMap map_ckv64,
                       const __grid_constant__ CUtensorMap map_kr32,
                       const __grid_constant__ CUtensorMap map_sc,
                       const __grid_constant__ CUtensorMap map_q, const DecodeArgs args) {
    using namespace pair;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t base = ptx::smem_u32(smem_raw);
    if (base & 1023u) {   // swizzled operands need a 1 KB aligned base; uniform over the cluster
        if (threadIdx.x == 0) record_error(kErrUnsupported);
        return;
    }
    uint8_t *smem = smem_raw;
    Misc *misc = reinterpret_cast<Misc *>(smem + OFF_MISC);
    volatile int32_t *abort_flag = &misc->abort_flag;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = ptx::cluster_ctarank();      // 0 = leader
    const int64_t part = blockIdx.x >> 1;
    const int64_t P = args.num_parts;

    auto bar = [&](const uint64_t *b) { return ptx::smem_u32(b); };
    // address of a barrier of the leader CTA, as seen from this CTA
    auto leader_bar = [&](const uint64_t *b) { return ptx::mapa(ptx::smem_u32(b), 0); };

    // ---------------------------------------------------------------- setup
    if (threadIdx.x == 0) {
        // E4M3: a slot is full once the eight dequantising warps of the pair
        // have widened it (and, for QK^T, the leader's k_R copies have landed)
        for (int i = 0; i < QK_STAGES; ++i) {
            ptx::mbar_init(bar(&misc->qk_full[i]), kFp8 ? 9 : 1);
            ptx::mbar_init(bar(&misc->qk_empty[i]), 1);
            if (kFp8) ptx::mbar_init(bar(&misc->code_qk[i]), 1);
        }
        for (int i = 0; i < PV_STAGES; ++i) {
            ptx::mbar_init(bar(&misc->pv_full[i]), kFp8 ? 8 : 1);
            ptx::mbar_init(bar(&misc->pv_empty[i]), 1);
            ptx::mbar_init(bar(&misc->pv_landed[i]), 1);
            if (kFp8) ptx::mbar_init(bar(&misc->code_pv[i]), 1);
        }
        for (int i = 0; i < NSB; ++i) ptx::mbar_init(bar(&misc->s_full[i]), 1);
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(bar(&misc->p_ready[i]), 8);
            ptx::mbar_init(bar(&misc->pv_done[i]), 1);
        }
        ptx::mbar_init(bar(&misc->q_ready), 8);     // 4 segment warps x 2 CTAs
        ptx::mbar_init(bar(&misc->o_free), 8);      // 4 segment warps x 2 CTAs
        ptx::mbar_init(bar(&misc->drain), 1);
        ptx::mbar_init(bar(&misc->q_free), 1);      // multicast commit from the leader
        ptx::mbar_init(bar(&misc->seg_done), 4);    // 4 softmax warps
        ptx::mbar_init(bar(&misc->q_tma), 1);
        ptx::mbar_init(bar(&misc->q_stage_free), 4);   // this CTA's 4 segment warps
        misc->abort_flag = 0;
        ptx::fence_mbar_init();
    }
    for (int i = threadIdx.x; i < 3 * 128; i += blockDim.x)
        (i < 256 ? misc->xtag[i >> 7][i & 127] : misc->xltag[i - 256]) = 1u;   // tag of "use -1"
    if (warp == 1) {
        ptx::tmem_alloc<2>(bar(reinterpret_cast<uint64_t *>(&misc->tmem_base)), TMEM_COLS);
        ptx::tmem_relinquish<2>();
    }
    ptx::grid_dep_launch();
    // The plan reads only the sequence lengths and the block table, which no
    // kernel of a decode step writes (the kernel ahead on the stream produces
    // q): it is made, down to this partition's first segment and that
    // segment's first page ids, before waiting for that kernel.
    if (warp == 0) {
        const SeqCursor c = find_sequence(args.seq_lens, args.batch, args.max_pages, args.n_q, TOK,
                                          P, -1);
        const int64_t N = c.total;   // plan cost
        const int64_t ts = (part < c.parts) ? part_start(part, N, c.parts) : N;
        const SeqCursor s = find_sequence(args.seq_lens, args.batch, args.max_pages, args.n_q, TOK,
                                          P, ts);
        SegmentWalker w0;
        w0.seq_lens = args.seq_lens;
        w0.batch = args.batch;
        w0.max_pages = args.max_pages;
        w0.n_q = args.n_q;
        w0.tile_tokens = TOK;
        w0.N = N;
        w0.P = c.parts;
        w0.p = part;
        w0.b = s.b;
        w0.O = s.cost_off;
        w0.S = s.slot_base;
        w0.tile = (part < c.parts) ? part_start(part, N, c.parts) : 0;
        w0.te = (part < c.parts) ? part_start(part + 1, N, c.parts) : 0;
        const bool have0 = w0.next();
        if (lane == 0) {
            misc->cur_b = w0.b;
            misc->cur_O = w0.O;
            misc->cur_S = w0.S;
            misc->cur_N = N;
            misc->cur_P = c.parts;
            misc->first_tile = w0.tile;
            misc->first_slot = have0 ? w0.slot : 0;
            misc->first_b = have0 ? w0.seg_b : -1;
            misc->first_L = have0 ? w0.L : 0;
            misc->first_t_begin = have0 ? static_cast<int32_t>(w0.t_begin) : 0;
            misc->first_t_end = have0 ? static_cast<int32_t>(w0.t_end) : 0;
            if (have0) {   // the first page numbers, for the producers
                const int32_t *trow0 = args.block_table + static_cast<int64_t>(w0.seg_b) * args.max_pages;
                int32_t *pg = reinterpret_cast<int32_t *>(smem + OFF_FIRST_PAGES);
#pragma unroll
                for (int i = 0; i < FIRST_PAGES; ++i)
                    pg[i] = (w0.t_begin + i < w0.t_end) ? trow0[w0.t_begin + i] : 0;
            }
            ptx::prefetch_tensormap(&map_ckv32);
            ptx::prefetch_tensormap(&map_ckv64);
            ptx::prefetch_tensormap(&map_kr32);
            if (kFp8) ptx::prefetch_tensormap(&map_sc);
            else ptx::prefetch_tensormap(&map_q);
        }
    }
    ptx::grid_dep_wait();   // other global memory from here on
    ptx::tc_fence_before();
    __syncthreads();
    ptx::cluster_sync();
    ptx::tc_fence_after();
    const uint32_t tmem = misc->tmem_base;

    SegmentWalker walk;
    walk.seq_lens = args.seq_lens;
    walk.batch = args.batch;
    walk.max_pages = args.max_pages;
    walk.n_q = args.n_q;
    walk.tile_tokens = TOK;
    walk.N = misc->cur_N;
    walk.P = misc->cur_P;
    walk.p = part;
    walk.b = misc->cur_b;
    walk.O = misc->cur_O;
    walk.S = misc->cur_S;
    walk.te = (part < walk.P) ? part_start(part + 1, walk.N, walk.P) : 0;   // 0: idle partition
    walk.tile = misc->first_tile;
    walk.primed = misc->first_b >= 0;
    walk.seg_b = misc->first_b;
    walk.L = misc->first_L;
    walk.t_begin = misc->first_t_begin;
    walk.t_end = misc->first_t_end;
    walk.slot = misc->first_slot;

    if (warp == 0 || warp == 6) {
        // ------------------------------------------------------ TMA producers
        // warp 0 fills the QK^T ring (own 32 tokens x 9 channel blocks), warp 6
        // the P.V ring (64 tokens x this SM's 4 channel blocks). Completion of
        // both CTAs' copies is counted on the leader's barriers. E4M3: the c_KV
        // codes of a slot land on this CTA's own barrier (code_qk / code_pv) for
        // the dequantising warps; k_R (bf16) still lands on the leader's.
        const bool qk = (warp == 0);
        if (ptx::elect_one()) {
            uint64_t *fullb = qk ? misc->qk_full : misc->pv_full;
            uint64_t *emptyb = qk ? misc->qk_empty : misc->pv_empty;
            uint64_t *codeb = qk ? misc->code_qk : misc->code_pv;
            const int nst = qk ? QK_STAGES : PV_STAGES;
            const uint32_t tx = kFp8 ? 2 * (OWN * 128) : 2 * (qk ? STAGE_QK : STAGE_PV);
            int64_t k = 0;
            bool bad_page = false;
            if (!kFp8 && qk && walk.primed) {
                // the first segment's Q: blocks 0..QT-1 to the staging area (the
                // segment warps move them to tensor memory), the rest to their place.
                // (The E4M3 kernel loads it like any other segment's: at its
                // 128-register cap the staged path made the dequantising warps spill.)
                const uint32_t qbar = bar(&misc->q_tma);
                ptx::mbar_arrive_expect_tx(qbar, NB * ROWS_CTA * 128);
                for (int j = 0; j < NB; ++j)
                    ptx::tma_load_3d(j < QT ? base + OFF_QSTAGE + j * (ROWS_CTA * 128)
                                            : base + OFF_Q + (j - QT) * (ROWS_CTA * 128),
                                     &map_q, qbar, 64 * j, ROWS_CTA * static_cast<int>(rank), walk.seg_b);
            }
            bool first_seg = walk.primed;
            for (; !*abort_flag && walk.next(); first_seg = false) {
                const int32_t *trow = args.block_table + static_cast<int64_t>(walk.seg_b) * args.max_pages;
                for (int64_t t = walk.t_begin; t < walk.t_end; ++t, ++k) {
                    const int s = static_cast<int>(k % nst);
                    const int64_t use = k / nst;
                    // the first tiles' pages were read with the plan (k counts the
                    // first segment's tiles first)
                    int32_t page = (first_seg && k < FIRST_PAGES)
                                       ? reinterpret_cast<const int32_t *>(smem + OFF_FIRST_PAGES)[k]
                                       : trow[t];
                    if (page < 0 || page >= args.num_pages) { bad_page = true; page = 0; }
                    if (use >= 1 && !wait_bounded(bar(&emptyb[s]), (use - 1) & 1, abort_flag,
                                                  args.timeout_ns))
                        break;
                    if (!kFp8 && !qk && k == 1 &&   // slot 1 held the first segment's staged Q
                        !wait_bounded(bar(&misc->q_stage_free), 0, abort_flag, args.timeout_ns))
                        break;
                    const uint32_t fb = (rank == 0) ? bar(&fullb[s]) : leader_bar(&fullb[s]);
                    if constexpr (kFp8) {
                        // codes, then 32 tokens' scales for each dequantising warp
                        // into that warp's last row of block 3 (QK^T) or 1 (P.V)
                        const uint32_t cb = bar(&codeb[s]);
                        ptx::mbar_arrive_expect_tx(cb, CODE_BYTES + SC_BYTES);
                        if (qk) {
                            const uint32_t st = base + OFF_QK + s * STAGE_QK;
                            for (int i = 0; i < 4; ++i)   // [32 own tokens x 128 codes] boxes
                                ptx::tma_load_3d(st + CODE_OFF + i * (OWN * 128), &map_ckv32, cb, 128 * i,
                                                 OWN * rank, page);
                            for (int w = 0; w < 4; ++w)   // dequantising warp w: row 8w + 7 of block 3
                                ptx::tma_load_2d(st + 3 * (OWN * 128) + (8 * w + 7) * 128, &map_sc, cb,
                                                 OWN * rank, page);
                            if (rank == 0) ptx::mbar_arrive_expect_tx(fb, tx);
                            ptx::tma_load_3d_pair(st + 8 * (OWN * 128), &map_kr32, fb, 0, OWN * rank, page);
                        } else {
                            const uint32_t st = base + OFF_PV + s * STAGE_PV;
                            for (int v = 0; v < 2; ++v)   // this SM's channels 256v + 128 rank + [0, 128)
                                for (int h = 0; h < 2; ++h)
                                    ptx::tma_load_3d(st + CODE_OFF + v * (TOK * 128) + h * (OWN * 128),
                                                     &map_ckv32, cb, 256 * v + 128 * static_cast<int>(rank),
                                                     OWN * h, page);
                            for (int w = 0; w < 4; ++w)   // dequantising warp w: row 16w + 15 of block 1
                                ptx::tma_load_2d(st + 1 * (TOK * 128) + (16 * w + 15) * 128, &map_sc, cb,
                                                 OWN * (w >> 1), page);
                        }
                        continue;
                    }
                    if (rank == 0) ptx::mbar_arrive_expect_tx(fb, tx);
                    if (qk) {
                        const uint32_t st = base + OFF_QK + s * STAGE_QK;
                        for (int j = 0; j < 8; ++j)
                            ptx::tma_load_3d_pair(st + j * (OWN * 128), &map_ckv32, fb, 64 * j,
                                                  OWN * rank, page);
                        ptx::tma_load_3d_pair(st + 8 * (OWN * 128), &map_kr32, fb, 0, OWN * rank, page);
                    } else {
                        const uint32_t st = base + OFF_PV + s * STAGE_PV;
                        for (int u = 0; u < 4; ++u) {
                            const int blk = 4 * (u >> 1) + 2 * static_cast<int>(rank) + (u & 1);
                            ptx::tma_load_3d_pair(st + u * (TOK * 128), &map_ckv64, fb, 64 * blk, 0,
                                                  page);
                        }
                    }
                }
            }
            if (bad_page) record_error(kErrDeviceBounds);
            // drain: the leader waits until every issued slot has landed
            // (E4M3: each CTA waits for its own code copies)
            if (kFp8) {
                for (int64_t kk = (k >= nst ? k - nst : 0); kk < k; ++kk)
                    wait_bounded<false>(bar(&codeb[kk % nst]), (kk / nst) & 1, abort_flag, args.timeout_ns);
            } else if (rank == 0) {
                for (int64_t kk = (k >= nst ? k - nst : 0); kk < k; ++kk)
                    wait_bounded(bar(&fullb[kk % nst]), (kk / nst) & 1, abort_flag, args.timeout_ns);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------ MMA issuer (leader)
        // Two cursors: QK^T of tile kq and P.V of tile kp (kp < kq <= kp + 3,
        // three score buffers). Whichever is ready is issued; the polls are
        // non-blocking so a late KV tile never holds back a ready P.V.
        if (rank == 0 && ptx::elect_one()) {
            SegmentWalker wq = walk, wp = walk;
            bool q_has = wq.next(), p_has = wp.next();
            int64_t tq = q_has ? wq.t_begin : 0, tp = p_has ? wp.t_begin : 0;
            int64_t kq = 0, kp = 0, gq = 0, gp = 0;
            bool q_ready_seen = false, o_free_seen = false;
            bool landed_sent = false;   // landing of P.V slot kp forwarded to both CTAs
            uint64_t idle_since = ptx::globaltimer_ns();
            uint32_t spins = 0;
            while ((q_has || p_has) && !*abort_flag) {
                bool progressed = false;
                if (q_has && kq < kp + NSB) {
                    if (!q_ready_seen) q_ready_seen = ptx::mbar_test_wait(bar(&misc->q_ready), gq & 1);
                    const int s = static_cast<int>(kq % QK_STAGES);
                    const int sb = static_cast<int>(kq % NSB);   // score buffer: tile kq - 3's
                                                                  // P.V is issued (its softmax read it)
                    if (q_ready_seen &&
                        ptx::mbar_test_wait(bar(&misc->qk_full[s]), (kq / QK_STAGES) & 1)) {
                        ptx::tc_fence_after();
                        // descriptors advance by (byte offset >> 4) in the start-address field
                        const uint64_t a0 = ptx::smem_desc(base + OFF_Q, 16, 1024, ptx::kSwizzle128B);
                        const uint64_t b0 = ptx::smem_desc(base + OFF_QK + s * STAGE_QK, 16, 1024,
                                                           ptx::kSwizzle128B);
                        const uint32_t d = tmem + TMEM_S + 32 * sb;
#pragma unroll
                        for (int j = 0; j < NB; ++j) {
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk) {
                                const uint64_t b = b0 + ((j * (OWN * 128) + kk * 32) >> 4);
                                const uint32_t acc = (j | kk) ? 1u : 0u;
                                if (j < QT)   // A from tensor memory: 8 columns per 16-channel step
                                    ptx::mma_bf16_ts<2>(d, tmem + TMEM_Q + 32 * j + 8 * kk, b, IDESC_QK,
                                                        acc);
                                else
                                    ptx::mma_bf16_ss<2>(
                                        d, a0 + (((j - QT) * (ROWS_CTA * 128) + kk * 32) >> 4), b,
                                        IDESC_QK, acc);
                            }
                        }
                        ptx::mma_commit_pair(bar(&misc->qk_empty[s]), 0x3);
                        ptx::mma_commit_pair(bar(&misc->s_full[sb]), 0x3);
                        ++kq;
                        if (++tq == wq.t_end) {
                            // the segment's last QK^T: once done, its Q may be replaced
                            ptx::mma_commit_pair(bar(&misc->q_free), 0x3);
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
                    const int s = static_cast<int>(kp & 1);            // P buffer
                    const int ps = static_cast<int>(kp % PV_STAGES);   // P.V operand slot
                    // Once both CTAs' copies of slot ps have landed, say so to each
                    // CTA: the softmax warps clear the rows past a sequence's end in
                    // its last tile before they report P ready.
                    if (!landed_sent &&
                        ptx::mbar_test_wait(bar(&misc->pv_full[ps]), (kp / PV_STAGES) & 1)) {
                        ptx::mbar_arrive(bar(&misc->pv_landed[ps]));
                        ptx::mbar_arrive_cluster(ptx::mapa(bar(&misc->pv_landed[ps]), 1));
                        landed_sent = true;
                        progressed = true;
                    }
                    if (landed_sent && (!first || gp == 0 || o_free_seen) &&
                        ptx::mbar_test_wait(bar(&misc->p_ready[s]), (kp >> 1) & 1)) {
                        landed_sent = false;
                        ptx::tc_fence_after();
                        const uint64_t a0 = ptx::smem_desc(base + OFF_P + s * P_BYTES, 16, 1024,
                                                           ptx::kSwizzle128B);
                        const uint64_t b0 = ptx::smem_desc(base + OFF_PV + ps * STAGE_PV, TOK * 128,
                                                           1024, ptx::kSwizzle128B);
#pragma unroll
                        for (int c = 0; c < 2; ++c) {
#pragma unroll
                            for (int kk = 0; kk < TOK / 16; ++kk) {
                                ptx::mma_bf16_ss<2>(tmem + TMEM_O + 128 * c, a0 + ((kk * 32) >> 4),
                                                    b0 + (((2 * c) * (TOK * 128) + kk * 2048) >> 4),
                                                    IDESC_PV, (first && kk == 0) ? 0u : 1u);
                            }
                        }
                        ptx::mma_commit_pair(bar(&misc->pv_empty[ps]), 0x3);
                        ptx::mma_commit_pair(bar(&misc->pv_done[s]), 0x3);
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
            // every MMA issued so far has finished before tensor memory is freed
            ptx::mma_commit_pair(bar(&misc->drain), 0x1);
            wait_bounded<false>(bar(&misc->drain), 0, abort_flag, args.timeout_ns);
        }
    } else if (kFp8 && warp >= kDqWarp0) {
        // ------------------------------------------------------ dequantising warps
        if constexpr (kFp8) {
            const int dq = warp - kDqWarp0;
            // every warp takes 8 of a QK^T slot's 32 rows and 16 of a P.V slot's
            // 64, converting QK^T one tile ahead of P.V (the MMAs consume them in
            // that order); the scale copies hold the CTA's 32 QK^T tokens and
            // P.V tokens 32 (dq / 2) + [0, 32)
            TileCursor cq, cp;
            cq.w = walk;
            cq.start();
            cp = cq;
            int64_t kq = 0, kp = 0;
            bool ok = true;
            auto qk_tile = [&]() {
                ok = dequant_tile<4, 1>(cq, kq, args, base + OFF_QK, STAGE_QK, OWN * 128, QK_STAGES, misc->code_qk,
                                        misc->qk_full, 8 * dq, 0, OWN * static_cast<int>(rank), rank, lane,
                                        abort_flag);
                cq.advance();
                ++kq;
            };
            if (cq.have) qk_tile();
            while (ok && cp.have && !*abort_flag) {
                if (cq.have) qk_tile();
                if (!ok) break;
                ok = dequant_tile<2, 2>(cp, kp, args, base + OFF_PV, STAGE_PV, TOK * 128, PV_STAGES, misc->code_pv,
                                        misc->pv_full, 16 * dq, 32 * (dq >> 1), 0, rank, lane, abort_flag);
                cp.advance();
                ++kp;
            }
        }
    } else if (warp >= kSegWarp0) {
        // ------------------------------------------------------ segment warps
        // One warp per tensor-memory lane quadrant. At a segment's start they
        // load its Q; when the last QK^T of a segment is done they load the next
        // segment's Q, and when its last P.V is done they write its partial
        // result -- so neither sits on the softmax warps' path from one tile to
        // the next.
        const int q4 = warp & 3;                       // TMEM lane quadrant
        const int lt = q4 * 32 + lane;                 // TMEM lane 0..127
        const int row = lt & 63;                       // local query row
        const int half = lt >> 6;                      // which 128 channels of each MMA's 256
        const int grow = ROWS_CTA * static_cast<int>(rank) + row;  // row within the sequence
        const bool real_row = grow < args.rows;
        const uint32_t lane_base = static_cast<uint32_t>(q4 * 32) << 16;
        const int st_tid = threadIdx.x - kSegWarp0 * 32;   // 0..127
        auto arrive_leader = [&](uint64_t *b) {
            __syncwarp();
            if (lane == 0) {
                if (rank == 0) ptx::mbar_arrive(bar(b));
                else ptx::mbar_arrive_cluster(leader_bar(b));
            }
        };
        // Q of sequence b: channel blocks 0..5 into tensor memory in the
        // duplicated 2-SM A layout (this lane holds row lt % 64, so lanes lt and
        // lt ^ 64 carry the same row), blocks 6..8 into shared memory
        // (128-byte swizzled, K-major).
        // The loads are issued in three rounds of independent requests (half of
        // the shared-memory blocks with each of the first two), so a segment
        // start costs three global-load latencies rather than one per block.
        auto load_q = [&](int32_t b) {
            const __nv_bfloat16 *qb = args.q + static_cast<int64_t>(b) * args.rows * D;
            const __nv_bfloat16 *qrow = qb + static_cast<int64_t>(real_row ? grow : 0) * D;
            constexpr int NSM = ROWS_CTA * (NB - QT) * 8 / 128 / 2;   // 8 + 8 chunks of blocks 5..8
#pragma unroll 1
            for (int j0 = 0; j0 < QT; j0 += 2) {   // up to two 64-channel blocks per round
                const int nj = (j0 + 1 < QT) ? 2 : 1;
                uint4 v[16], sv[NSM];
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    v[i] = (real_row && (i < 8 || nj == 2)) ? ld_global_nc_v4(qrow + 64 * j0 + 8 * i)
                                                            : make_uint4(0, 0, 0, 0);
                if (j0 < 4) {
#pragma unroll
                    for (int i = 0; i < NSM; ++i) {
                        const int idx = st_tid + 128 * (i + NSM * (j0 >> 1));
                        const int r = idx / ((NB - QT) * 8);
                        const int cc = idx - r * ((NB - QT) * 8);   // 16-byte chunk among blocks 5..8
                        const int gr = ROWS_CTA * static_cast<int>(rank) + r;
                        sv[i] = (gr < args.rows)
                                    ? ld_global_nc_v4(qb + static_cast<int64_t>(gr) * D + 64 * QT + cc * 8)
                                    : make_uint4(0, 0, 0, 0);
                    }
#pragma unroll
                    for (int i = 0; i < NSM; ++i) {
                        const int idx = st_tid + 128 * (i + NSM * (j0 >> 1));
                        const int r = idx / ((NB - QT) * 8);
                        const int cc = idx - r * ((NB - QT) * 8);
                        st_shared_v4(base + OFF_Q + (cc >> 3) * (ROWS_CTA * 128) + sw128(r, cc & 7), sv[i].x,
                                     sv[i].y, sv[i].z, sv[i].w);
                    }
                }
#pragma unroll
                for (int jj = 0; jj < 2; ++jj) {
                    if (jj >= nj) break;
                    uint32_t w[32];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        w[4 * i] = v[8 * jj + i].x;
                        w[4 * i + 1] = v[8 * jj + i].y;
                        w[4 * i + 2] = v[8 * jj + i].z;
                        w[4 * i + 3] = v[8 * jj + i].w;
                    }
                    ptx::tmem_st32(tmem + lane_base + TMEM_Q + 32 * (j0 + jj), w);
                }
            }
            ptx::tmem_wait_st();
            ptx::fence_proxy_async_smem();
            ptx::tc_fence_before();
            arrive_leader(&misc->q_ready);
        };

        // The first segment's Q, landed by TMA: blocks QT..8 are in place,
        // blocks 0..QT-1 (128-byte swizzled rows) are copied to tensor memory.
        auto load_q_staged = [&]() {
            if (wait_bounded(bar(&misc->q_tma), 0, abort_flag, args.timeout_ns)) {
#pragma unroll 1
                for (int j = 0; j < QT; ++j) {
                    uint32_t w[32];
                    const uint32_t src = base + OFF_QSTAGE + j * (ROWS_CTA * 128);
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const uint4 v = ld_shared_v4(src + sw128(row, i));
                        w[4 * i] = v.x;
                        w[4 * i + 1] = v.y;
                        w[4 * i + 2] = v.z;
                        w[4 * i + 3] = v.w;
                    }
                    ptx::tmem_st32(tmem + lane_base + TMEM_Q + 32 * j, w);
                }
            }
            ptx::tmem_wait_st();
            ptx::fence_proxy_async_smem();
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(bar(&misc->q_stage_free));
            arrive_leader(&misc->q_ready);
        };

        auto prefetch_q = [&](int32_t b) {   // the next segment's Q rows into L2
            if (!real_row || half) return;
            const char *qrow = reinterpret_cast<const char *>(
                args.q + (static_cast<int64_t>(b) * args.rows + grow) * D);
#pragma unroll
            for (int i = 0; i < D * 2 / 128; ++i)
                asm volatile("prefetch.global.L2 [%0];" ::"l"(qrow + 128 * i));
        };

        int64_t k = 0;
        int64_t g = 0;
        bool have = walk.next();
        if (have) {
            if constexpr (kFp8) load_q(walk.seg_b);
            else load_q_staged();
        }
        while (have && !*abort_flag) {
            const int64_t slot = walk.slot;
            const int64_t kl = k + (walk.t_end - walk.t_begin) - 1;   // the segment's last tile
            k = kl + 1;
            have = walk.next();
            if (have) {
                prefetch_q(walk.seg_b);
                // the next segment's Q, once the last QK^T of this one is done
                if (!wait_bounded<false>(bar(&misc->q_free), g & 1, abort_flag, args.timeout_ns)) break;
                ptx::tc_fence_after();
                load_q(walk.seg_b);
            }
            // this segment's partial result, once its last P.V is done
            if (!wait_bounded<false>(bar(&misc->seg_done), g & 1, abort_flag, args.timeout_ns)) break;
            if (!wait_bounded<false>(bar(&misc->pv_done[kl & 1]), (kl >> 1) & 1, abort_flag,
                                     args.timeout_ns))
                break;
            ptx::tc_fence_after();
            const float l_row = misc->seg_l[g & 1][row];
            const float m_run = misc->seg_m[g & 1][row];
            const float inv = (l_row > 0.f) ? 1.f / l_row : 0.f;
            // O / l of this lane's row, 8 columns at a time through a 1 KB
            // shared-memory tile ([32 rows x 32 B], 16-byte chunks XOR-swizzled
            // by row), so that each global store instruction writes 16 rows x 32
            // contiguous bytes instead of 32 rows x 16 bytes
            const uint32_t stg = base + OFF_EPI + static_cast<uint32_t>(warp - kSegWarp0) * 1024u;
            const int rr = lane >> 1, rc = lane & 1;   // read-back: rows rr + 16i, chunk rc
#pragma unroll 1
            for (int cch = 0; cch < 8; ++cch) {
                uint32_t o[32];
                ptx::tmem_ld32(tmem + lane_base + TMEM_O + 32 * cch, o);
                ptx::tmem_wait_ld();
                // column 32*cch of MMA c = cch/4 holds channel 256c + 128*half + 32*(cch%4)
                const int ch = 256 * (cch >> 2) + 128 * half + 32 * (cch & 3);
#pragma unroll
                for (int pc = 0; pc < 4; ++pc) {
                    __syncwarp();   // the previous piece has been read back
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        const int j = 8 * pc + 4 * c;
                        st_shared_v4(stg + lane * 32 + ((c ^ ((lane >> 2) & 1)) << 4),
                                     __float_as_uint(__uint_as_float(o[j]) * inv),
                                     __float_as_uint(__uint_as_float(o[j + 1]) * inv),
                                     __float_as_uint(__uint_as_float(o[j + 2]) * inv),
                                     __float_as_uint(__uint_as_float(o[j + 3]) * inv));
                    }
                    __syncwarp();
#pragma unroll
                    for (int i = 0; i < 2; ++i) {
                        const int r = rr + 16 * i;                        // staging row = lane r of this warp
                        const int grow_r = ROWS_CTA * static_cast<int>(rank) + ((q4 * 32 + r) & 63);
                        const uint4 v = ld_shared_v4(stg + r * 32 + ((rc ^ ((r >> 2) & 1)) << 4));
                        if (grow_r < args.rows)
                            *reinterpret_cast<uint4 *>(args.o_part + (slot * args.rows + grow_r) * DC + ch +
                                                       8 * pc + 4 * rc) = v;
                    }
                }
            }
            if (real_row && half == 0) {
                args.lse_part[slot * args.rows + grow] =
                    (l_row > 0.f) ? m_run * args.scale + logf(l_row) : -INFINITY;
            }
            ptx::tc_fence_before();
            arrive_leader(&misc->o_free);
            ++g;
        }
    } else {
        // ------------------------------------------------------ softmax
        const int q4 = warp & 3;                       // TMEM lane quadrant
        const int lt = q4 * 32 + lane;                 // TMEM lane 0..127
        const int row = lt & 63;                       // local query row
        const int half = lt >> 6;                      // which 32 tokens of the tile
        const int grow = ROWS_CTA * static_cast<int>(rank) + row;  // row within the sequence
        const bool real_row = grow < args.rows;
        const int qi = real_row ? grow / args.heads : 0;
        const uint32_t lane_base = static_cast<uint32_t>(q4 * 32) << 16;
        const int st_tid = threadIdx.x - kSoftmaxWarp0 * 32;   // 0..127
        auto arrive_leader = [&](uint64_t *b) {
            __syncwarp();
            if (lane == 0) {
                if (rank == 0) ptx::mbar_arrive(bar(b));
                else ptx::mbar_arrive_cluster(leader_bar(b));
            }
        };
        int64_t k = 0;
        int64_t seg_no = 0;
        bool have = walk.next();
        while (have && !*abort_flag) {
            const int32_t seg_b = walk.seg_b;
            const int32_t L = walk.L;
            const int64_t slot = walk.slot;
            const int64_t k0 = k;
            const int64_t t_begin = walk.t_begin, t_end = walk.t_end;
            const int32_t vis = real_row ? (L - args.n_q + qi + 1) : 0;
            float m_run = -INFINITY;      // running max (raw score units)
            float l_run = 0.f;            // this lane's share of the row sum
            bool ok = true;
            for (int64_t t = t_begin; t < t_end; ++t, ++k) {
                const int s = static_cast<int>(k & 1);          // P buffer, exchange words
                const int sb = static_cast<int>(k % NSB);       // score buffer
                if (!wait_bounded<false>(bar(&misc->s_full[sb]), (k / NSB) & 1, abort_flag,
                                         args.timeout_ns)) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                uint32_t sr[32];
                ptx::tmem_ld32(tmem + lane_base + TMEM_S + 32 * sb, sr);
                ptx::tmem_wait_ld();

                const int32_t tok0 = static_cast<int32_t>(t) * TOK + half * OWN;
                float v[32];
                if (tok0 + 32 <= vis) {   // every token of this half visible: no mask
#pragma unroll
                    for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(sr[j]);
                } else {
#pragma unroll
                    for (int j = 0; j < 32; ++j) v[j] = (tok0 + j < vis) ? __uint_as_float(sr[j]) : -INFINITY;
                }
                float mx = max_of<32>(v);
                // Half-row maxima meet through tagged words: the lowest mantissa
                // bit carries the parity of the word's use (k / 2); a lane cannot
                // be two uses ahead of its partner's read (it needs the partner's
                // word of every tile in between), so one bit tells the uses apart.
                // Both lanes use the same two values with that bit cleared (1 ulp,
                // so the exponentials stay finite for scores up to ~2^23 / scale_log2).
                const uint32_t tag = static_cast<uint32_t>((k >> 1) & 1);
                const uint32_t mine = (__float_as_uint(mx) & ~1u) | tag;
                reinterpret_cast<volatile uint32_t *>(misc->xtag[s])[lt] = mine;
                uint32_t other = 0;
                if (!wait_word(&misc->xtag[s][lt ^ 64], tag, abort_flag, args.timeout_ns, &other)) {
                    ok = false;
                    break;
                }
                mx = fmaxf(__uint_as_float(mine & ~1u), __uint_as_float(other & ~1u));

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
                l_run = fmaf(l_run, alpha, (ps[0] + ps[1]) + (ps[2] + ps[3]));

                // rescale the accumulated O rows held by this lane
                const bool need = (k > k0) && (alpha != 1.f);
                const bool any_need = __any_sync(0xffffffffu, need);
                if (any_need) {
                    const int64_t kp = k - 1;
                    if (!wait_bounded<false>(bar(&misc->pv_done[kp & 1]), (kp >> 1) & 1, abort_flag,
                                             args.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after();
#pragma unroll 1
                    for (int cch = 0; cch < 8; ++cch) {
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
                // P buffer s is free once the value product of tile k - 2 is done
                if (k >= 2 && !wait_bounded<false>(bar(&misc->pv_done[s]), ((k >> 1) - 1) & 1,
                                                   abort_flag, args.timeout_ns)) {
                    ok = false;
                    break;
                }
                const uint32_t pb = base + OFF_P + s * P_BYTES;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    st_shared_v4(pb + sw128(row, 4 * half + c),
                                 pack_bf16x2(v[8 * c + 0], v[8 * c + 1]),
                                 pack_bf16x2(v[8 * c + 2], v[8 * c + 3]),
                                 pack_bf16x2(v[8 * c + 4], v[8 * c + 5]),
                                 pack_bf16x2(v[8 * c + 6], v[8 * c + 7]));
                }
                // Last tile of the sequence: the page's rows past its end were loaded
                // with the page and may hold any bits (an unwritten or recycled page
                // slot). Their P is 0, but 0 * NaN = NaN in the value product, so
                // they are cleared in this CTA's P.V slot once it has landed.
                const int32_t valid = L - static_cast<int32_t>(t) * TOK;
                if (!kFp8 && valid < TOK) {   // (E4M3: the dequantising warps wrote zeros there)
                    const int ps = static_cast<int>(k % PV_STAGES);
                    if (!wait_bounded(bar(&misc->pv_landed[ps]), (k / PV_STAGES) & 1, abort_flag,
                                      args.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    const uint32_t slot_base = base + OFF_PV + ps * STAGE_PV;
                    const int n16 = (TOK - valid) * 8;   // 16-byte chunks per channel block
                    for (int idx = st_tid; idx < 4 * n16; idx += 128) {
                        const int u = idx / n16, rem = idx - u * n16;
                        st_shared_v4(slot_base + u * (TOK * 128) + (valid + (rem >> 3)) * 128 +
                                         (rem & 7) * 16,
                                     0u, 0u, 0u, 0u);
                    }
                }
                ptx::fence_proxy_async_smem();
                if (any_need) ptx::tc_fence_before();   // order the O rescale stores
                arrive_leader(&misc->p_ready[s]);
            }
            if (!ok) break;

            // the segment's row sum: both halves of the row meet; published with
            // the running maximum for the segment warps' epilogue
            const uint32_t ltag = static_cast<uint32_t>(seg_no & 1);   // (as above, by segment)
            const int gpar = static_cast<int>(seg_no & 1);
            ++seg_no;
            const uint32_t lmine = (__float_as_uint(l_run) & ~1u) | ltag;
            reinterpret_cast<volatile uint32_t *>(misc->xltag)[lt] = lmine;
            uint32_t lother = 0;
            if (!wait_word(&misc->xltag[lt ^ 64], ltag, abort_flag, args.timeout_ns, &lother)) break;
            // identical in both lanes: the same two truncated terms, added commutatively
            const float l_row = __uint_as_float(lmine & ~1u) + __uint_as_float(lother & ~1u);
            if (half == 0) {
                misc->seg_l[gpar][row] = l_row;
                misc->seg_m[gpar][row] = m_run;
            }
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(bar(&misc->seg_done));
            (void)seg_b;
            (void)slot;
            have = walk.next();
        }
    }

    // ---------------------------------------------------------------- teardown
    ptx::tc_fence_before();
    __syncthreads();
    ptx::cluster_sync();
    ptx::tc_fence_after();
    if (warp == 1) ptx::tmem_dealloc<2>(tmem, TMEM_COLS);
}

// ===========================================================================
// Single-CTA kernel: d_c = 64, d_R = 8 (RoPE padded to 16 in shared memory)
// ===========================================================================
namespace single {
constexpr int DC = 64, DR = 8, D = DC + DR;
constexpr int ROWS = 128;
constexpr int TOK = 128;                        // tokens per tile (two pages)
constexpr uint32_t Q_LAT = ROWS * 128;          // 16384: [128 rows x 64 ch] swizzled
constexpr uint32_t Q_ROPE = ROWS * 16;          // 2048: [128 rows x 8 ch] core matrices
constexpr uint32_t Q_BYTES = Q_LAT + 2 * Q_ROPE;          // + zero K-chunk
constexpr uint32_t ST_LAT = TOK * 128;                    // 16384
constexpr uint32_t ST_ROPE = TOK * 16;                    // 2048
constexpr uint32_t STAGE_BYTES = ST_LAT + 2 * ST_ROPE;    // 20480
#ifndef MLA_SINGLE_STAGES
#define MLA_SINGLE_STAGES 4
#endif
constexpr int STAGES = MLA_SINGLE_STAGES;                 // KV ring depth (score and P buffers: 2)
constexpr uint32_t P_BYTES = 2 * ROWS * 128;              // [128 rows x 128 tok] = 2 K-blocks
constexpr uint32_t OFF_Q = 0;
constexpr uint32_t OFF_STAGE = 20480;                     // Q rounded up to 1 KB multiple
constexpr uint32_t OFF_P = OFF_STAGE + STAGES * STAGE_BYTES;
constexpr uint32_t OFF_MISC = OFF_P + 2 * P_BYTES;
constexpr uint32_t SMEM_BYTES = OFF_MISC + pair::MISC_BYTES + 1024;  // + alignment slack
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TMEM_O = 0;                            // 64 columns
constexpr uint32_t TMEM_S = 128;                          // two 128-column score buffers
constexpr uint32_t IDESC_QK = ptx::idesc_bf16(128, TOK, 0, 0);
constexpr uint32_t IDESC_PV = ptx::idesc_bf16(128, DC, 0, 1);
static_assert(Q_BYTES <= OFF_STAGE, "q");
static_assert(STAGES >= 2 && STAGES <= 8, "ring");
static_assert(SMEM_BYTES <= 232448, "smem");
static_assert((OFF_P % 1024) == 0 && (OFF_MISC % 1024) == 0, "align");
}  // namespace single

template <bool kSplit>
__global__ void __launch_bounds__(kDecodeThreads, 1)
    decode_single_kernel(const __grid_constant__ CUtensorMap map_ckv,
                         const __grid_constant__ CUtensorMap map_kr, const DecodeArgs args) {
    using namespace single;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_base = ptx::smem_u32(smem_raw);
    const uint32_t base = (raw_base + 1023u) & ~1023u;
    uint8_t *smem = smem_raw + (base - raw_base);
    Misc *misc = reinterpret_cast<Misc *>(smem + OFF_MISC);
    volatile int32_t *abort_flag = &misc->abort_flag;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t part = blockIdx.x;
    const int64_t P = args.num_parts;
    auto bar = [&](const uint64_t *b) { return ptx::smem_u32(b); };

    if (threadIdx.x == 0) {
        for (int i = 0; i < STAGES; ++i) {
            ptx::mbar_init(bar(&misc->kv_full[i]), 1);
            ptx::mbar_init(bar(&misc->kv_empty[i]), 1);
        }
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(bar(&misc->s_full[i]), 1);
            ptx::mbar_init(bar(&misc->s_free[i]), 4);
            ptx::mbar_init(bar(&misc->p_ready[i]), 4);
            ptx::mbar_init(bar(&misc->pv_done[i]), 1);
        }
        ptx::mbar_init(bar(&misc->q_ready), 4);
        ptx::mbar_init(bar(&misc->o_free), 4);
        ptx::mbar_init(bar(&misc->drain), 1);
        misc->abort_flag = 0;
        ptx::fence_mbar_init();
    }
    // zero the stages and Q (so never-loaded rows and the padded RoPE K-chunk
    // hold zeros rather than stale bit patterns)
    for (uint32_t off = threadIdx.x * 16; off < OFF_MISC; off += kDecodeThreads * 16)
        st_shared_v4(base + off, 0, 0, 0, 0);
    ptx::fence_proxy_async_smem();
    if (warp == 1) {
        ptx::tmem_alloc<1>(bar(reinterpret_cast<uint64_t *>(&misc->tmem_base)), TMEM_COLS);
        ptx::tmem_relinquish<1>();
    }
    ptx::grid_dep_launch();
    // The plan reads only the sequence lengths, which no kernel of a decode step
    // writes: it is made, down to this partition's first segment, before
    // waiting for the kernel ahead on the stream (which produces q).
    if (warp == 0) {
        const SeqCursor c = find_sequence(args.seq_lens, args.batch, args.max_pages, args.n_q, TOK,
                                          P, -1);
        const int64_t N = c.total;   // plan cost
        const int64_t ts = (part < c.parts) ? part_start(part, N, c.parts) : N;
        const SeqCursor s = find_sequence(args.seq_lens, args.batch, args.max_pages, args.n_q, TOK,
                                          P, ts);
        SegmentWalker w0;
        w0.seq_lens = args.seq_lens;
        w0.batch = args.batch;
        w0.max_pages = args.max_pages;
        w0.n_q = args.n_q;
        w0.tile_tokens = TOK;
        w0.N = N;
        w0.P = c.parts;
        w0.p = part;
        w0.b = s.b;
        w0.O = s.cost_off;
        w0.S = s.slot_base;
        w0.tile = (part < c.parts) ? part_start(part, N, c.parts) : 0;
        w0.te = (part < c.parts) ? part_start(part + 1, N, c.parts) : 0;
        const bool have0 = w0.next();
        if (lane == 0) {
            misc->cur_b = w0.b;
            misc->cur_O = w0.O;
            misc->cur_S = w0.S;
            misc->cur_N = N;
            misc->cur_P = c.parts;
            misc->first_tile = w0.tile;
            misc->first_slot = have0 ? w0.slot : 0;
            misc->first_b = have0 ? w0.seg_b : -1;
            misc->first_L = have0 ? w0.L : 0;
            misc->first_t_begin = have0 ? static_cast<int32_t>(w0.t_begin) : 0;
            misc->first_t_end = have0 ? static_cast<int32_t>(w0.t_end) : 0;
            if (have0)   // the first page numbers, for the producer (a hint: L2 only)
                asm volatile("prefetch.global.L2 [%0];" ::"l"(
                    args.block_table + static_cast<int64_t>(w0.seg_b) * args.max_pages + 2 * w0.t_begin));
            ptx::prefetch_tensormap(&map_ckv);
            ptx::prefetch_tensormap(&map_kr);
        }
    }
    ptx::grid_dep_wait();   // other global memory from here on
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = misc->tmem_base;

    SegmentWalker walk;
    walk.seq_lens = args.seq_lens;
    walk.batch = args.batch;
    walk.max_pages = args.max_pages;
    walk.n_q = args.n_q;
    walk.tile_tokens = TOK;
    walk.N = misc->cur_N;
    walk.P = misc->cur_P;
    walk.p = part;
    walk.b = misc->cur_b;
    walk.O = misc->cur_O;
    walk.S = misc->cur_S;
    walk.te = (part < walk.P) ? part_start(part + 1, walk.N, walk.P) : 0;   // 0: idle partition
    walk.tile = misc->first_tile;
    walk.primed = misc->first_b >= 0;   // every role starts from the published first segment
    walk.seg_b = misc->first_b;
    walk.L = misc->first_L;
    walk.t_begin = misc->first_t_begin;
    walk.t_end = misc->first_t_end;
    walk.slot = misc->first_slot;

    if (warp == 0) {
        if (ptx::elect_one()) {
            int64_t k = 0;
            bool bad_page = false;
            while (!*abort_flag && walk.next()) {
                const int32_t *trow = args.block_table + static_cast<int64_t>(walk.seg_b) * args.max_pages;
                const int32_t npages = (walk.L + 63) / 64;
                for (int64_t t = walk.t_begin; t < walk.t_end; ++t, ++k) {
                    const int s = static_cast<int>(k % STAGES);
                    const int32_t p0 = static_cast<int32_t>(2 * t);
                    const bool two = p0 + 1 < npages;
                    int32_t pg[2] = {trow[p0], two ? trow[p0 + 1] : 0};
                    for (int i = 0; i < 2; ++i)
                        if (pg[i] < 0 || pg[i] >= args.num_pages) { bad_page = true; pg[i] = 0; }
                    if (k >= STAGES && !wait_bounded(bar(&misc->kv_empty[s]), ((k / STAGES) - 1) & 1,
                                                     abort_flag, args.timeout_ns))
                        break;
                    const uint32_t fb = bar(&misc->kv_full[s]);
                    const uint32_t npg = two ? 2u : 1u;
                    ptx::mbar_arrive_expect_tx(fb, npg * (64 * 128 + 64 * 16));
                    const uint32_t st = base + OFF_STAGE + s * STAGE_BYTES;
                    for (uint32_t i = 0; i < npg; ++i) {
                        ptx::tma_load_3d(st + i * (64 * 128), &map_ckv, fb, 0, 0, pg[i]);
                        ptx::tma_load_3d(st + ST_LAT + i * (64 * 16), &map_kr, fb, 0, 0, pg[i]);
                    }
                }
            }
            if (bad_page) record_error(kErrDeviceBounds);
            for (int64_t kk = (k >= STAGES ? k - STAGES : 0); kk < k; ++kk)
                wait_bounded(bar(&misc->kv_full[kk % STAGES]), (kk / STAGES) & 1, abort_flag, args.timeout_ns);
        }
    } else if (warp == 1) {
        if (ptx::elect_one()) {
            int64_t k = 0, g = 0;
            bool ok = true;
            auto issue_pv = [&](int64_t kp, bool first_of_seg) -> bool {
                const int s = static_cast<int>(kp & 1);            // P buffer
                const int ks = static_cast<int>(kp % STAGES);      // KV stage
                if (!wait_bounded(bar(&misc->p_ready[s]), (kp >> 1) & 1, abort_flag, args.timeout_ns))
                    return false;
                ptx::tc_fence_after();
                const uint32_t st = base + OFF_STAGE + ks * STAGE_BYTES;
                const uint32_t pbuf = base + OFF_P + s * P_BYTES;
                for (int kk = 0; kk < TOK / 16; ++kk) {
                    const uint64_t a = ptx::smem_desc(pbuf + (kk >> 2) * (ROWS * 128) + (kk & 3) * 32,
                                                      16, 1024, ptx::kSwizzle128B);
                    const uint64_t b = ptx::smem_desc(st + kk * 2048, 8192, 1024, ptx::kSwizzle128B);
                    ptx::mma_bf16_ss<1>(tmem + TMEM_O, a, b, IDESC_PV,
                                        (first_of_seg && kk == 0) ? 0u : 1u);
                }
                ptx::mma_commit(bar(&misc->kv_empty[ks]));
                ptx::mma_commit(bar(&misc->pv_done[s]));
                return true;
            };
            while (ok && !*abort_flag && walk.next()) {
                const int64_t k0 = k;
                if (!wait_bounded(bar(&misc->q_ready), g & 1, abort_flag, args.timeout_ns)) break;
                for (int64_t t = walk.t_begin; t < walk.t_end; ++t, ++k) {
                    const int s = static_cast<int>(k & 1);             // score buffer
                    const int ks = static_cast<int>(k % STAGES);       // KV stage
                    if (!wait_bounded(bar(&misc->kv_full[ks]), (k / STAGES) & 1, abort_flag,
                                      args.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    if (k >= 2 && !wait_bounded(bar(&misc->s_free[s]), ((k >> 1) - 1) & 1,
                                                abort_flag, args.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after();
                    const uint32_t st = base + OFF_STAGE + ks * STAGE_BYTES;
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint64_t a = ptx::smem_desc(base + OFF_Q + kk * 32, 16, 1024,
                                                          ptx::kSwizzle128B);
                        const uint64_t b = ptx::smem_desc(st + kk * 32, 16, 1024, ptx::kSwizzle128B);
                        ptx::mma_bf16_ss<1>(tmem + TMEM_S + TOK * s, a, b, IDESC_QK, kk ? 1u : 0u);
                    }
                    {   // RoPE step: 8 real channels + 8 zero channels, no swizzle
                        const uint64_t a = ptx::smem_desc(base + OFF_Q + Q_LAT, Q_ROPE, 128,
                                                          ptx::kSwizzleNone);
                        const uint64_t b = ptx::smem_desc(st + ST_LAT, ST_ROPE, 128, ptx::kSwizzleNone);
                        ptx::mma_bf16_ss<1>(tmem + TMEM_S + TOK * s, a, b, IDESC_QK, 1u);
                    }
                    ptx::mma_commit(bar(&misc->s_full[s]));
                    if (k > k0) {
                        if (k - 1 == k0 && g > 0) {
                            if (!wait_bounded(bar(&misc->o_free), (g - 1) & 1, abort_flag,
                                              args.timeout_ns)) {
                                ok = false;
                                break;
                            }
                        }
                        if (!issue_pv(k - 1, k - 1 == k0)) { ok = false; break; }
                    }
                }
                if (!ok) break;
                if (k - 1 == k0 && g > 0) {
                    if (!wait_bounded(bar(&misc->o_free), (g - 1) & 1, abort_flag, args.timeout_ns))
                        break;
                }
                if (!issue_pv(k - 1, k - 1 == k0)) break;
                ++g;
            }
            ptx::mma_commit(bar(&misc->drain));
            wait_bounded(bar(&misc->drain), 0, abort_flag, args.timeout_ns);
        }
    } else {
        // kSplit (at most 64 query rows): query row r sits in MMA rows
        // 32 (r / 16) + r % 16 and the same + 16, both TMEM lanes of one warp;
        // the first lane takes the tile's tokens 0..63, the second 64..127, and
        // the two meet by shuffles (row maximum per tile, sums and O at the
        // end). Otherwise MMA row = query row and a lane takes all 128 tokens.
        constexpr int TT = kSplit ? TOK / 2 : TOK;      // tokens per thread and tile
        const int q4 = warp & 3;
        const int tl = q4 * 32 + lane;                  // TMEM lane = MMA row
        const int half = kSplit ? (lane >> 4) : 0;
        const int row = kSplit ? 16 * q4 + (lane & 15) : tl;   // query row
        const bool real_row = row < args.rows;
        const bool warp_real = (kSplit ? 16 * q4 : 32 * q4) < args.rows;   // warp holds a real row
        const int qi = real_row ? row / args.heads : 0;
        const uint32_t lane_base = static_cast<uint32_t>(q4 * 32) << 16;
        const int st_tid = threadIdx.x - kSoftmaxWarp0 * 32;
        auto arrive = [&](uint64_t *b) {
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(bar(b));
        };
        auto load_q = [&](int32_t b) {   // all of a thread's loads in flight at once
            const __nv_bfloat16 *qb = args.q + static_cast<int64_t>(b) * args.rows * D;
            constexpr int QR = kSplit ? ROWS / 2 : ROWS;              // query rows held
            constexpr int NQ = (QR * (D / 8) + 127) / 128;           // chunks per thread
            uint4 v[NQ];
#pragma unroll
            for (int i = 0; i < NQ; ++i) {
                const int idx = st_tid + 128 * i;
                const int r = idx / (D / 8);
                const int cc = idx - r * (D / 8);
                v[i] = (r < args.rows) ? ld_global_nc_v4(qb + static_cast<int64_t>(r) * D + cc * 8)
                                       : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int i = 0; i < NQ; ++i) {
                const int idx = st_tid + 128 * i;
                if (idx >= QR * (D / 8)) break;
                const int r = idx / (D / 8);
                const int cc = idx - r * (D / 8);
#pragma unroll
                for (int dup = 0; dup < (kSplit ? 2 : 1); ++dup) {
                    const int m = kSplit ? 32 * (r >> 4) + (r & 15) + 16 * dup : r;   // MMA row
                    uint32_t dst;
                    if (cc < 8) dst = base + OFF_Q + sw128(m, cc);
                    else dst = base + OFF_Q + Q_LAT + (m >> 3) * 128 + (m & 7) * 16;
                    st_shared_v4(dst, v[i].x, v[i].y, v[i].z, v[i].w);
                }
            }
            ptx::fence_proxy_async_smem();
            arrive(&misc->q_ready);
        };

        int64_t k = 0;
        bool have = walk.next();
        if (have) load_q(walk.seg_b);
        while (have && !*abort_flag) {
            const int32_t L = walk.L;
            const int64_t slot = walk.slot;
            const int64_t k0 = k;
            const int64_t t_begin = walk.t_begin, t_end = walk.t_end;
            const int32_t vis = real_row ? (L - args.n_q + qi + 1) : 0;
            float m_run = -INFINITY, l_run = 0.f;
            bool ok = true;
            for (int64_t t = t_begin; t < t_end; ++t, ++k) {
                const int s = static_cast<int>(k & 1);
                if (!wait_bounded(bar(&misc->s_full[s]), (k >> 1) & 1, abort_flag, args.timeout_ns)) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                float v[TT];
                if (warp_real) {
                    // (a tensor-memory load takes one column address for the whole
                    // warp: with kSplit every lane loads both halves and keeps its own)
#pragma unroll
                    for (int c = 0; c < TT / 32; ++c) {
                        uint32_t sr[32];
                        ptx::tmem_ld32(tmem + lane_base + TMEM_S + TOK * s + 32 * c, sr);
                        if (kSplit) {
                            uint32_t sr2[32];
                            ptx::tmem_ld32(tmem + lane_base + TMEM_S + TOK * s + TT + 32 * c, sr2);
                            ptx::tmem_wait_ld();
#pragma unroll
                            for (int j = 0; j < 32; ++j) v[32 * c + j] = __uint_as_float(half ? sr2[j] : sr[j]);
                        } else {
                            ptx::tmem_wait_ld();
#pragma unroll
                            for (int j = 0; j < 32; ++j) v[32 * c + j] = __uint_as_float(sr[j]);
                        }
                    }
                }
                ptx::tc_fence_before();
                arrive(&misc->s_free[s]);

                float alpha = 1.f;
                if (warp_real) {
                    const int32_t tok0 = static_cast<int32_t>(t) * TOK + TT * half;
                    if (tok0 + TT > vis) {   // mask the tokens this row does not see
#pragma unroll
                        for (int j = 0; j < TT; ++j) v[j] = (tok0 + j < vis) ? v[j] : -INFINITY;
                    }
                    float mx = max_of<TT>(v);
                    if (kSplit) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));   // the row's two halves
                    if (mx > -INFINITY && (m_run == -INFINITY ||
                                           (mx - m_run) * args.scale_log2 > kRescaleThreshold)) {
                        alpha = (m_run == -INFINITY) ? 0.f : exp2f((m_run - mx) * args.scale_log2);
                        m_run = mx;
                    }
                    const float mb = (m_run == -INFINITY) ? 0.f : m_run * args.scale_log2;
                    float psum = 0.f;
#pragma unroll
                    for (int j = 0; j < TT; ++j) {
                        v[j] = exp2f(fmaf(v[j], args.scale_log2, -mb));
                        psum += v[j];
                    }
                    l_run = fmaf(l_run, alpha, psum);   // (kSplit: this half's share)
                }
                const bool need = warp_real && (k > k0) && (alpha != 1.f);
                if (__any_sync(0xffffffffu, need)) {
                    const int64_t kp = k - 1;
                    if (!wait_bounded(bar(&misc->pv_done[kp & 1]), (kp >> 1) & 1, abort_flag,
                                      args.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after();
#pragma unroll 1
                    for (int cch = 0; cch < DC / 32; ++cch) {
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
                    const int64_t kp = k - 2;
                    if (!wait_bounded(bar(&misc->pv_done[kp & 1]), (kp >> 1) & 1, abort_flag,
                                      args.timeout_ns)) {
                        ok = false;
                        break;
                    }
                }
                if (warp_real) {
                    // this thread's tokens of MMA row tl (kSplit: one 64-token K block;
                    // the other block of the row keeps the zeros written at start)
                    const uint32_t pb = base + OFF_P + s * P_BYTES + half * (ROWS * 128);
#pragma unroll
                    for (int c = 0; c < TT / 8; ++c) {
                        st_shared_v4(pb + (c >> 3) * (ROWS * 128) + sw128(tl, c & 7),
                                     pack_bf16x2(v[8 * c + 0], v[8 * c + 1]),
                                     pack_bf16x2(v[8 * c + 2], v[8 * c + 3]),
                                     pack_bf16x2(v[8 * c + 4], v[8 * c + 5]),
                                     pack_bf16x2(v[8 * c + 6], v[8 * c + 7]));
                    }
                }
                // Last tile of the sequence: the stage's c_KV rows past its end (the
                // tail of the last page, or a second page not loaded for this tile)
                // may hold any bits; P is 0 there, but 0 * NaN = NaN in the value
                // product, so they are cleared. QK^T of this tile has finished
                // reading the stage (s_full) and P.V waits for p_ready.
                const int32_t valid = L - static_cast<int32_t>(t) * TOK;
                if (valid < TOK) {
                    const uint32_t st = base + OFF_STAGE + static_cast<int>(k % STAGES) * STAGE_BYTES;
                    for (int idx = st_tid; idx < (TOK - valid) * 8; idx += 128)
                        st_shared_v4(st + (valid + (idx >> 3)) * 128 + (idx & 7) * 16, 0u, 0u, 0u, 0u);
                }
                ptx::fence_proxy_async_smem();
                ptx::tc_fence_before();
                arrive(&misc->p_ready[s]);
            }
            if (!ok) break;
            have = walk.next();
            if (have) load_q(walk.seg_b);
            const int64_t kl = k - 1;
            if (!wait_bounded(bar(&misc->pv_done[kl & 1]), (kl >> 1) & 1, abort_flag,
                              args.timeout_ns))
                break;
            ptx::tc_fence_after();
            if (warp_real) {
                // kSplit: the row's sum and O are its two lanes' shares added (the
                // same sum in both lanes); each lane writes one 32-channel half
                const float l_row = kSplit ? l_run + __shfl_xor_sync(0xffffffffu, l_run, 16) : l_run;
                const float inv = (l_row > 0.f) ? 1.f / l_row : 0.f;
                float *dst = args.o_part + (slot * args.rows + row) * DC;
#pragma unroll 1
                for (int cch = 0; cch < DC / 32; ++cch) {
                    uint32_t o[32];
                    ptx::tmem_ld32(tmem + lane_base + TMEM_O + 32 * cch, o);
                    ptx::tmem_wait_ld();
                    if (kSplit) {
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            const float mine = __uint_as_float(o[j]);
                            const float other = __shfl_xor_sync(0xffffffffu, mine, 16);
                            o[j] = __float_as_uint(half ? other + mine : mine + other);   // lane order: tokens 0..63 first
                        }
                    }
                    if (real_row && (!kSplit || cch == half)) {
                        float4 *d4 = reinterpret_cast<float4 *>(dst + 32 * cch);
#pragma unroll
                        for (int j = 0; j < 8; ++j)
                            d4[j] = make_float4(__uint_as_float(o[4 * j]) * inv,
                                                __uint_as_float(o[4 * j + 1]) * inv,
                                                __uint_as_float(o[4 * j + 2]) * inv,
                                                __uint_as_float(o[4 * j + 3]) * inv);
                    }
                }
                if (real_row && half == 0)
                    args.lse_part[slot * args.rows + row] =
                        (l_row > 0.f) ? m_run * args.scale + logf(l_row) : -INFINITY;
            }
            ptx::tc_fence_before();
            arrive(&misc->o_free);
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    if (warp == 1) ptx::tmem_dealloc<1>(tmem, TMEM_COLS);
}

}  // namespace mla
