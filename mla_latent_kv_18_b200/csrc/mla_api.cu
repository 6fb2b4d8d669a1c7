// Host side of the C ABI declared in include/mla_decode.h: argument
// validation, tensor-map construction, the partition plan and kernel launches.
// Everything is asynchronous on the caller's stream; no device memory is
// allocated here.
#include <cmath>
#include <cstdint>
#include <cstring>
#include <algorithm>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>

#include "mla_decode.h"
#include "common.cuh"
#include "decode.cuh"
#include "small_kernels.cuh"
#include "prefill.cuh"

namespace {

using mla::kErrCuda;
using mla::kErrInvalidArg;
using mla::kErrUnsupported;

constexpr int64_t kDefaultTimeoutNs = 2000000000LL;   // 2 s per bounded wait
constexpr int kMaxDevices = 64;

enum class Variant { Pair512, Single64, None };

Variant variant_of(const mla_dims *d) {
    if (d->d_latent == 512 && d->d_rope == 64) return Variant::Pair512;
    if (d->d_latent == 64 && d->d_rope == 8) return Variant::Single64;
    return Variant::None;
}

int tile_tokens(Variant v) { return v == Variant::Pair512 ? mla::pair::TOK : mla::single::TOK; }

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Validates the dims common to every call; returns MLA_OK or an error.
mla_status check_dims(const mla_dims *d, bool need_variant) {
    if (!d) return MLA_ERR_INVALID_ARG;
    if (d->num_heads <= 0 || d->n_q <= 0 || d->d_nope <= 0 || d->d_latent <= 0 || d->d_rope <= 0 ||
        d->d_v <= 0 || d->page_size <= 0)
        return MLA_ERR_INVALID_ARG;
    if ((d->d_nope % 8) || (d->d_latent % 8) || (d->d_rope % 8) || (d->d_v % 8))
        return MLA_ERR_UNSUPPORTED;
    if (need_variant) {
        if (variant_of(d) == Variant::None) return MLA_ERR_UNSUPPORTED;
        if (d->page_size != 64) return MLA_ERR_UNSUPPORTED;
        if (static_cast<int64_t>(d->n_q) * d->num_heads > 128) return MLA_ERR_UNSUPPORTED;
    }
    return MLA_OK;
}

float scale_of(const mla_dims *d) {
    return d->softmax_scale > 0.f ? d->softmax_scale
                                  : static_cast<float>(1.0 / std::sqrt(double(d->d_nope + d->d_rope)));
}

constexpr int32_t kGatherMaxWidth = 512;

// Per-device one-time state: capability check and kernel attributes.
struct DeviceState {
    std::once_flag once;
    mla_status status = MLA_OK;
    int sms = 0;   // multiprocessor count
};
DeviceState g_dev[kMaxDevices];

int device_sms() {   // after device_ready() succeeded
    int dev = 0;
    return (cudaGetDevice(&dev) == cudaSuccess && dev >= 0 && dev < kMaxDevices) ? g_dev[dev].sms : 0;
}

mla_status device_ready() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MLA_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return MLA_ERR_UNSUPPORTED;
    DeviceState &st = g_dev[dev];
    std::call_once(st.once, [&] {
        cudaDeviceProp prop;
        if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) { st.status = MLA_ERR_CUDA; return; }
        if (prop.major != 10 || prop.minor != 0) { st.status = MLA_ERR_UNSUPPORTED; return; }
        st.sms = prop.multiProcessorCount;
        if (cudaFuncSetAttribute(mla::decode_pair_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 mla::pair::SMEM_BYTES) != cudaSuccess ||
            cudaFuncSetAttribute(mla::decode_pair_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 mla::pair::SMEM_BYTES) != cudaSuccess ||
            cudaFuncSetAttribute(mla::decode_single_kernel<false>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 mla::single::SMEM_BYTES) != cudaSuccess ||
            cudaFuncSetAttribute(mla::decode_single_kernel<true>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 mla::single::SMEM_BYTES) != cudaSuccess ||
            cudaFuncSetAttribute(mla::proj_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 mla::proj_smem_bytes(256)) != cudaSuccess ||
            cudaFuncSetAttribute(mla::gather_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 64 * kGatherMaxWidth * 2) != cudaSuccess ||
            cudaFuncSetAttribute(mla::combine_out_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 mla::co_smem_bytes(128, mla::kCoMaxNT, mla::kCoMaxSlots)) != cudaSuccess ||
            cudaFuncSetAttribute(mla::decompress_kernel<false>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 mla::dkv::SMEM_BYTES) != cudaSuccess ||
            cudaFuncSetAttribute(mla::decompress_kernel<true>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 mla::dkv::SMEM_BYTES) != cudaSuccess ||
            cudaFuncSetAttribute(mla::prefill_attn_kernel,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 mla::pfa::SMEM_BYTES) != cudaSuccess) {
            st.status = MLA_ERR_CUDA;
            return;
        }
        // The decode step's kernels keep the same (largest) shared-memory
        // carve-out, so an SM does not reconfigure between them.
        const int carve = cudaSharedmemCarveoutMaxShared;
        if (cudaFuncSetAttribute(mla::proj_tc_kernel, cudaFuncAttributePreferredSharedMemoryCarveout, carve) !=
                cudaSuccess ||
            cudaFuncSetAttribute(mla::combine_kernel, cudaFuncAttributePreferredSharedMemoryCarveout, carve) !=
                cudaSuccess ||
            cudaFuncSetAttribute(mla::combine_out_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 carve) != cudaSuccess ||
            cudaFuncSetAttribute(mla::decode_pair_kernel<false>, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 carve) != cudaSuccess ||
            cudaFuncSetAttribute(mla::decode_pair_kernel<true>, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 carve) != cudaSuccess ||
            cudaFuncSetAttribute(mla::decode_single_kernel<false>, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 carve) != cudaSuccess ||
            cudaFuncSetAttribute(mla::decode_single_kernel<true>, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 carve) != cudaSuccess) {
            st.status = MLA_ERR_CUDA;
            return;
        }
    });
    return st.status;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link
// dependency on libcuda).
using EncodeFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                              const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                              const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                              CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeFn encode_fn() {
    static EncodeFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeFn>(p);
    });
    return fn;
}

// 3-D bf16 map over a page pool: dims (channels, 64 tokens, pages).
mla_status pool_map(CUtensorMap *m, const mla_pool *pool, int32_t channels, int32_t num_pages,
                    uint32_t box_ch, uint32_t box_tok, CUtensorMapSwizzle sw) {
    EncodeFn enc = encode_fn();
    if (!enc) return MLA_ERR_CUDA;
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(channels), 64,
                                static_cast<cuuint64_t>(num_pages)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(pool->token_stride) * 2,
                                   static_cast<cuuint64_t>(pool->page_stride) * 2};
    const cuuint32_t box[3] = {box_ch, box_tok, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(pool->base), dims,
                     strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? MLA_OK : MLA_ERR_INVALID_ARG;
}

// Launch with programmatic stream serialization: the kernel may be scheduled
// while the kernel before it on the stream finishes; it waits for that
// kernel's completion (griddepcontrol.wait) before its first global-memory
// access, so only its launch and on-chip set-up overlap.
template <typename... KArgs, typename... Args>
mla_status launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                      Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, args...) == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

mla_status launch_status() {
    return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

// 3-D bf16 map with 128-byte swizzle: dims (d0 inner, d1, d2), byte strides s1, s2.
mla_status map_3d(CUtensorMap *m, const void *base, uint64_t d0, uint64_t d1, uint64_t d2,
                  uint64_t s1, uint64_t s2, uint32_t b0, uint32_t b1, uint32_t b2) {
    EncodeFn enc = encode_fn();
    if (!enc) return MLA_ERR_CUDA;
    const cuuint64_t dims[3] = {d0, d1, d2};
    const cuuint64_t strides[2] = {s1, s2};
    const cuuint32_t box[3] = {b0, b1, b2};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides,
                     box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? MLA_OK : MLA_ERR_INVALID_ARG;
}

// out[t, h, :n_cols] = x[t, h, :K] W[h] on tensor cores (+ RoPE copy when rope != null).
mla_status launch_proj(const void *x, const void *w, void *out, const void *rope, int32_t T,
                       int32_t H, int32_t K, int32_t n_cols, int32_t out_stride, int32_t d_rope,
                       cudaStream_t s, const int32_t *positions = nullptr, double log_theta = 0.0) {
    const int NT = T >= 256 ? 256 : ((T + 15) / 16) * 16;
    CUtensorMap mw, mx;
    mla_status st;
    if ((st = map_3d(&mw, w, n_cols, K, H, uint64_t(n_cols) * 2, uint64_t(K) * n_cols * 2, 64, 64,
                     1)) != MLA_OK)
        return st;
    if ((st = map_3d(&mx, x, K, H, T, uint64_t(K) * 2, uint64_t(H) * K * 2, 64, 1, NT)) != MLA_OK)
        return st;
    mla::ProjArgs a;
    a.out = static_cast<__nv_bfloat16 *>(out);
    a.rope = static_cast<const __nv_bfloat16 *>(rope);
    a.positions = positions;
    a.log_theta = log_theta;
    a.timeout_ns = kDefaultTimeoutNs;
    a.T = T;
    a.H = H;
    a.K = K;
    a.n_cols = n_cols;
    a.out_stride = out_stride;
    a.d_rope = d_rope;
    a.NT = NT;
    a.stages = std::min(mla::kProjStages, (K + 63) / 64);
    dim3 grid(H, (n_cols + 127) / 128, (T + NT - 1) / NT);
    return launch_pdl(mla::proj_tc_kernel, grid, dim3(128), mla::proj_smem_bytes(NT, a.stages), s, mw, mx,
                      a);
}

// 3-D uint8 map over an E4M3 code pool: dims (channels, 64 tokens, pages),
// unswizzled boxes of [box_tok tokens x box_ch codes].
mla_status code_pool_map(CUtensorMap *m, const mla_pool *pool, int32_t channels, int32_t num_pages,
                         uint32_t box_ch, uint32_t box_tok) {
    EncodeFn enc = encode_fn();
    if (!enc) return MLA_ERR_CUDA;
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(channels), 64,
                                static_cast<cuuint64_t>(num_pages)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(pool->token_stride),
                                   static_cast<cuuint64_t>(pool->page_stride)};
    const cuuint32_t box[3] = {box_ch, box_tok, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(pool->base), dims, strides,
                     box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? MLA_OK : MLA_ERR_INVALID_ARG;
}

// 2-D fp32 map over the per-token scales [pages, 64]: boxes of box_tok tokens of one page.
mla_status scale_map(CUtensorMap *m, const float *scales, int32_t num_pages, uint32_t box_tok) {
    EncodeFn enc = encode_fn();
    if (!enc) return MLA_ERR_CUDA;
    const cuuint64_t dims[2] = {64, static_cast<cuuint64_t>(num_pages)};
    const cuuint64_t strides[1] = {64 * sizeof(float)};
    const cuuint32_t box[2] = {box_tok, 1};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float *>(scales), dims, strides, box,
                     estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                     CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? MLA_OK : MLA_ERR_INVALID_ARG;
}

mla_status check_pool(const mla_pool *p, int32_t channels) {
    if (!p || !p->base) return MLA_ERR_INVALID_ARG;
    if (!aligned(p->base, 16)) return MLA_ERR_INVALID_ARG;
    if (p->token_stride < channels || p->page_stride < p->token_stride) return MLA_ERR_INVALID_ARG;
    if ((p->token_stride % 8) || (p->page_stride % 8)) return MLA_ERR_INVALID_ARG;
    return MLA_OK;
}

int64_t round_up(int64_t x, int64_t a) { return (x + a - 1) / a * a; }

}  // namespace

extern "C" {

const char *mla_status_string(int32_t s) {
    switch (s) {
        case MLA_OK: return "MLA_OK";
        case MLA_ERR_INVALID_ARG: return "MLA_ERR_INVALID_ARG";
        case MLA_ERR_UNSUPPORTED: return "MLA_ERR_UNSUPPORTED";
        case MLA_ERR_CUDA: return "MLA_ERR_CUDA";
        case MLA_ERR_DEVICE_BOUNDS: return "MLA_ERR_DEVICE_BOUNDS";
        case MLA_ERR_TIMEOUT: return "MLA_ERR_TIMEOUT";
        default: return "MLA_ERR_UNKNOWN";
    }
}

int32_t mla_decode_num_parts(const mla_dims *dims, int64_t total_tiles, int32_t num_sms) {
    if (check_dims(dims, true) != MLA_OK || num_sms <= 0) return 1;
    // d_latent 512: at least 8 tiles per partition, at most one partition per
    // CTA pair (more, shorter partitions cost more in the merge than they save
    // at small batches); d_latent 64: one tile per partition at least, one
    // partition per SM at most (measured: 4 x 8192 tokens 33.7 -> 17.1 us)
    const Variant v = variant_of(dims);
    const int64_t units = (v == Variant::Pair512) ? num_sms / 2 : num_sms;
    const int64_t min_tiles = (v == Variant::Pair512) ? 8 : 1;
    int64_t parts = (total_tiles + min_tiles - 1) / min_tiles;
    if (parts > units) parts = units;
    if (parts < 1) parts = 1;
    return static_cast<int32_t>(parts);
}

size_t mla_decode_workspace_bytes(const mla_dims *dims, int32_t batch, int32_t num_parts) {
    if (check_dims(dims, true) != MLA_OK || batch < 0 || num_parts <= 0) return 0;
    const int64_t slots = static_cast<int64_t>(batch) + num_parts;
    const int64_t R = static_cast<int64_t>(dims->n_q) * dims->num_heads;
    const int64_t o_bytes = round_up(slots * R * dims->d_latent * 4, 256);
    return static_cast<size_t>(o_bytes + round_up(slots * R * 4, 256));
}

int32_t mla_default_num_splits(const mla_dims *dims, int32_t batch, int32_t max_seq_len,
                               int32_t num_sms) {
    if (check_dims(dims, true) != MLA_OK || batch <= 0 || max_seq_len <= 0 || num_sms <= 0) return 1;
    const int64_t tiles = mla::tiles_of_len(max_seq_len, tile_tokens(variant_of(dims)));
    return mla_decode_num_parts(dims, static_cast<int64_t>(batch) * tiles, num_sms);
}

size_t mla_decode_workspace_size(const mla_dims *dims, int32_t batch, int32_t num_splits) {
    return mla_decode_workspace_bytes(dims, batch, num_splits);
}

int64_t mla_decode_plan(const mla_dims *dims, const int32_t *seq_lens_host,
                        int32_t max_pages_per_seq, int32_t batch, int32_t num_parts,
                        int32_t *part_first, int32_t *slot_count, int64_t *slot_base) {
    if (check_dims(dims, true) != MLA_OK || batch < 0 || num_parts <= 0 || max_pages_per_seq <= 0)
        return -1;
    if (batch > 0 && !seq_lens_host) return -1;
    const int T = tile_tokens(variant_of(dims));
    int64_t N = 0, NB = 0;
    bool bad = false;
    for (int32_t b = 0; b < batch; ++b) {
        const int64_t n =
            mla::tiles_of_len(mla::clamp_len(seq_lens_host[b], max_pages_per_seq, dims->n_q, &bad), T);
        N += n;
        NB += (n > 0);
    }
    const int64_t C = mla::plan_cost(N, NB, T);
    const int64_t P = mla::parts_in_use(num_parts, N);
    int64_t CO = 0, S = 0;   // cost offset of the next non-empty sequence, slots so far
    for (int32_t b = 0; b < batch; ++b) {
        const int64_t n =
            mla::tiles_of_len(mla::clamp_len(seq_lens_host[b], max_pages_per_seq, dims->n_q, &bad), T);
        int64_t pf = -1, cnt = 0;
        if (n > 0) {
            pf = mla::part_of_tile(CO, C, P);
            cnt = mla::part_of_tile(CO + n - 1, C, P) - pf + 1;
            CO += n + mla::switch_cost(T);
        }
        if (part_first) part_first[b] = static_cast<int32_t>(pf);
        if (slot_count) slot_count[b] = static_cast<int32_t>(cnt);
        if (slot_base) slot_base[b] = S;
        S += cnt;
    }
    return S;
}

mla_status mla_absorb_q(const mla_dims *dims, const void *q_c, const void *q_r, const void *w_uk,
                        void *q_out, int32_t num_tokens, void *stream) {
    mla_status st = check_dims(dims, false);
    if (st != MLA_OK) return st;
    if (num_tokens < 0) return MLA_ERR_INVALID_ARG;
    if (dims->d_nope > 4096 || dims->d_latent > 4096) return MLA_ERR_UNSUPPORTED;
    if (num_tokens == 0) return MLA_OK;
    if (!q_c || !q_r || !w_uk || !q_out) return MLA_ERR_INVALID_ARG;
    if (!aligned(q_c, 16) || !aligned(q_r, 16) || !aligned(w_uk, 16) || !aligned(q_out, 16))
        return MLA_ERR_INVALID_ARG;
    if ((st = device_ready()) != MLA_OK) return st;
    return launch_proj(q_c, w_uk, q_out, q_r, num_tokens, dims->num_heads, dims->d_nope,
                       dims->d_latent, dims->d_latent + dims->d_rope, dims->d_rope,
                       static_cast<cudaStream_t>(stream));
}

mla_status mla_absorb_q_rope(const mla_dims *dims, const void *q_c, const void *q_r,
                             const void *w_uk, const int32_t *positions, float rope_theta,
                             void *q_out, int32_t num_tokens, void *stream) {
    mla_status st = check_dims(dims, false);
    if (st != MLA_OK) return st;
    if (num_tokens < 0 || !(rope_theta > 1.f) || !std::isfinite(rope_theta)) return MLA_ERR_INVALID_ARG;
    if (dims->d_nope > 4096 || dims->d_latent > 4096) return MLA_ERR_UNSUPPORTED;
    if (num_tokens == 0) return MLA_OK;
    if (!q_c || !q_r || !w_uk || !q_out || !positions) return MLA_ERR_INVALID_ARG;
    if (!aligned(q_c, 16) || !aligned(q_r, 16) || !aligned(w_uk, 16) || !aligned(q_out, 16) ||
        !aligned(positions, 4))
        return MLA_ERR_INVALID_ARG;
    if ((st = device_ready()) != MLA_OK) return st;
    return launch_proj(q_c, w_uk, q_out, q_r, num_tokens, dims->num_heads, dims->d_nope,
                       dims->d_latent, dims->d_latent + dims->d_rope, dims->d_rope,
                       static_cast<cudaStream_t>(stream), positions,
                       std::log(static_cast<double>(rope_theta)));
}

mla_status mla_absorb_out(const mla_dims *dims, const void *o_lat, const void *w_uv, void *out,
                          int32_t num_tokens, void *stream) {
    mla_status st = check_dims(dims, false);
    if (st != MLA_OK) return st;
    if (num_tokens < 0) return MLA_ERR_INVALID_ARG;
    if (dims->d_latent > 4096 || dims->d_v > 4096) return MLA_ERR_UNSUPPORTED;
    if (num_tokens == 0) return MLA_OK;
    if (!o_lat || !w_uv || !out) return MLA_ERR_INVALID_ARG;
    if (!aligned(o_lat, 16) || !aligned(w_uv, 16) || !aligned(out, 16)) return MLA_ERR_INVALID_ARG;
    if ((st = device_ready()) != MLA_OK) return st;
    return launch_proj(o_lat, w_uv, out, nullptr, num_tokens, dims->num_heads, dims->d_latent,
                       dims->d_v, dims->d_v, 0, static_cast<cudaStream_t>(stream));
}

}  // extern "C"

namespace {
// The split-KV arguments common to both cache formats (validated by the caller).
mla::DecodeArgs decode_args(const mla_dims *dims, const void *q, int32_t num_pages,
                            const int32_t *block_table, int32_t max_pages_per_seq,
                            const int32_t *seq_lens, int32_t batch, int32_t num_parts,
                            void *workspace) {
    const int64_t R = static_cast<int64_t>(dims->n_q) * dims->num_heads;
    const int64_t slots = static_cast<int64_t>(batch) + num_parts;
    mla::DecodeArgs a;
    a.q = static_cast<const __nv_bfloat16 *>(q);
    a.block_table = block_table;
    a.seq_lens = seq_lens;
    a.kv_scales = nullptr;
    a.o_part = static_cast<float *>(workspace);
    a.lse_part = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) +
                                           round_up(slots * R * dims->d_latent * 4, 256));
    a.timeout_ns = kDefaultTimeoutNs;
    a.max_pages = max_pages_per_seq;
    a.batch = batch;
    a.num_pages = num_pages;
    a.num_parts = num_parts;
    a.n_q = dims->n_q;
    a.heads = dims->num_heads;
    a.rows = static_cast<int32_t>(R);
    a.scale = scale_of(dims);
    a.scale_log2 = a.scale * 1.4426950408889634f;
    return a;
}

// q [batch, rows, 576] bf16 as [64 rows x 64 channels] boxes (128-byte swizzled):
// the pair kernel's TMA copy of a segment's Q; rows past `rows` read as zeros.
mla_status q_map(CUtensorMap *m, const void *q, const mla_dims *dims, int32_t batch) {
    const uint64_t D = static_cast<uint64_t>(dims->d_latent + dims->d_rope);
    const uint64_t R = static_cast<uint64_t>(dims->n_q) * dims->num_heads;
    return map_3d(m, q, D, R, static_cast<uint64_t>(batch), D * 2, R * D * 2, 64, mla::pair::ROWS_CTA, 1);
}

mla_status check_decode_common(const mla_dims *dims, const void *q, int32_t num_pages,
                               const int32_t *block_table, int32_t max_pages_per_seq,
                               const int32_t *seq_lens, int32_t batch, int32_t num_parts,
                               void *workspace, size_t workspace_bytes) {
    if (batch < 0 || num_parts <= 0 || max_pages_per_seq <= 0 || num_pages <= 0)
        return MLA_ERR_INVALID_ARG;
    if (batch == 0) return MLA_OK;
    if (!q || !block_table || !seq_lens || !workspace) return MLA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(block_table, 4) || !aligned(seq_lens, 4) ||
        !aligned(workspace, 256))
        return MLA_ERR_INVALID_ARG;
    if (workspace_bytes < mla_decode_workspace_bytes(dims, batch, num_parts)) return MLA_ERR_INVALID_ARG;
    return MLA_OK;
}
}  // namespace

extern "C" {

mla_status mla_decode_splitkv(const mla_dims *dims, const void *q, const mla_pool *ckv,
                              const mla_pool *kr, int32_t num_pages, const int32_t *block_table,
                              int32_t max_pages_per_seq, const int32_t *seq_lens, int32_t batch,
                              int32_t num_parts, void *workspace, size_t workspace_bytes,
                              void *stream) {
    mla_status st = check_dims(dims, true);
    if (st != MLA_OK) return st;
    if ((st = check_decode_common(dims, q, num_pages, block_table, max_pages_per_seq, seq_lens, batch,
                                  num_parts, workspace, workspace_bytes)) != MLA_OK)
        return st;
    if (batch == 0) return MLA_OK;
    if ((st = check_pool(ckv, dims->d_latent)) != MLA_OK) return st;
    if ((st = check_pool(kr, dims->d_rope)) != MLA_OK) return st;
    if ((st = device_ready()) != MLA_OK) return st;

    const mla::DecodeArgs a = decode_args(dims, q, num_pages, block_table, max_pages_per_seq, seq_lens,
                                          batch, num_parts, workspace);
    cudaStream_t s = static_cast<cudaStream_t>(stream);

    if (variant_of(dims) == Variant::Pair512) {
        CUtensorMap m32, m64, mkr;
        if ((st = pool_map(&m32, ckv, 512, num_pages, 64, mla::pair::OWN,
                           CU_TENSOR_MAP_SWIZZLE_128B)) != MLA_OK)
            return st;
        if ((st = pool_map(&m64, ckv, 512, num_pages, 64, mla::pair::TOK,
                           CU_TENSOR_MAP_SWIZZLE_128B)) != MLA_OK)
            return st;
        if ((st = pool_map(&mkr, kr, 64, num_pages, 64, mla::pair::OWN,
                           CU_TENSOR_MAP_SWIZZLE_128B)) != MLA_OK)
            return st;
        CUtensorMap mq;
        if ((st = q_map(&mq, q, dims, batch)) != MLA_OK) return st;
        return launch_pdl(mla::decode_pair_kernel<false>, dim3(2 * num_parts), dim3(mla::kPairThreads),
                          mla::pair::SMEM_BYTES, s, m32, m64, mkr, mkr /* no scales */, mq, a);
    } else {
        CUtensorMap mc, mkr;
        if ((st = pool_map(&mc, ckv, 64, num_pages, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B)) != MLA_OK)
            return st;
        if ((st = pool_map(&mkr, kr, 8, num_pages, 8, 64, CU_TENSOR_MAP_SWIZZLE_NONE)) != MLA_OK)
            return st;
        // at most 64 query rows: each row on two TMEM lanes, half the tile's tokens each
        return a.rows <= 64 ? launch_pdl(mla::decode_single_kernel<true>, dim3(num_parts), dim3(mla::kDecodeThreads),
                                         mla::single::SMEM_BYTES, s, mc, mkr, a)
                            : launch_pdl(mla::decode_single_kernel<false>, dim3(num_parts),
                                         dim3(mla::kDecodeThreads), mla::single::SMEM_BYTES, s, mc, mkr, a);
    }
}

mla_status mla_decode_splitkv_fp8(const mla_dims *dims, const void *q, const mla_pool *ckv8,
                                  const float *scales, const mla_pool *kr, int32_t num_pages,
                                  const int32_t *block_table, int32_t max_pages_per_seq,
                                  const int32_t *seq_lens, int32_t batch, int32_t num_parts,
                                  void *workspace, size_t workspace_bytes, void *stream) {
    mla_status st = check_dims(dims, true);
    if (st != MLA_OK) return st;
    if (variant_of(dims) != Variant::Pair512) return MLA_ERR_UNSUPPORTED;
    if ((st = check_decode_common(dims, q, num_pages, block_table, max_pages_per_seq, seq_lens, batch,
                                  num_parts, workspace, workspace_bytes)) != MLA_OK)
        return st;
    if (batch == 0) return MLA_OK;
    if (!ckv8 || !ckv8->base || !aligned(ckv8->base, 16) || ckv8->token_stride < dims->d_latent ||
        ckv8->page_stride < 64 * ckv8->token_stride || (ckv8->token_stride % 16) ||
        (ckv8->page_stride % 16))
        return MLA_ERR_INVALID_ARG;
    if (!scales || !aligned(scales, 16)) return MLA_ERR_INVALID_ARG;
    if ((st = check_pool(kr, dims->d_rope)) != MLA_OK) return st;
    if ((st = device_ready()) != MLA_OK) return st;

    mla::DecodeArgs a = decode_args(dims, q, num_pages, block_table, max_pages_per_seq, seq_lens, batch,
                                    num_parts, workspace);
    a.kv_scales = scales;
    CUtensorMap mc, mkr, msc;
    if ((st = code_pool_map(&mc, ckv8, 512, num_pages, 128, mla::pair::OWN)) != MLA_OK) return st;
    if ((st = pool_map(&mkr, kr, 64, num_pages, 64, mla::pair::OWN, CU_TENSOR_MAP_SWIZZLE_128B)) != MLA_OK)
        return st;
    if ((st = scale_map(&msc, scales, num_pages, 32)) != MLA_OK) return st;
    CUtensorMap mq;
    if ((st = q_map(&mq, q, dims, batch)) != MLA_OK) return st;
    return launch_pdl(mla::decode_pair_kernel<true>, dim3(2 * num_parts), dim3(mla::kPairThreadsFp8),
                      mla::pair::SMEM_BYTES, static_cast<cudaStream_t>(stream), mc, mc, mkr, msc, mq, a);
}

mla_status mla_combine(const mla_dims *dims, const void *workspace, size_t workspace_bytes,
                       const int32_t *seq_lens, int32_t max_pages_per_seq, int32_t batch,
                       int32_t num_parts, void *o_lat, float *lse_out, void *stream) {
    mla_status st = check_dims(dims, true);
    if (st != MLA_OK) return st;
    if (batch < 0 || num_parts <= 0 || max_pages_per_seq <= 0) return MLA_ERR_INVALID_ARG;
    if (batch == 0) return MLA_OK;
    if (!workspace || !seq_lens || !o_lat) return MLA_ERR_INVALID_ARG;
    if (!aligned(workspace, 256) || !aligned(o_lat, 16) || !aligned(seq_lens, 4) ||
        (lse_out && !aligned(lse_out, 4)))
        return MLA_ERR_INVALID_ARG;
    if (workspace_bytes < mla_decode_workspace_bytes(dims, batch, num_parts)) return MLA_ERR_INVALID_ARG;
    if ((st = device_ready()) != MLA_OK) return st;
    const int64_t R = static_cast<int64_t>(dims->n_q) * dims->num_heads;
    const int64_t slots = static_cast<int64_t>(batch) + num_parts;
    mla::CombineArgs a;
    a.o_part = static_cast<const float *>(workspace);
    a.lse_part = reinterpret_cast<const float *>(static_cast<const uint8_t *>(workspace) +
                                                 round_up(slots * R * dims->d_latent * 4, 256));
    a.seq_lens = seq_lens;
    a.o_lat = static_cast<__nv_bfloat16 *>(o_lat);
    a.lse_out = lse_out;
    a.batch = batch;
    a.max_pages = max_pages_per_seq;
    a.n_q = dims->n_q;
    a.rows = static_cast<int32_t>(R);
    a.d_c = dims->d_latent;
    a.tile_tokens = tile_tokens(variant_of(dims));
    a.num_parts = num_parts;
    dim3 grid(batch, static_cast<unsigned>((R + 3) / 4));
    return launch_pdl(mla::combine_kernel, grid, dim3(128), 0, static_cast<cudaStream_t>(stream), a);
}

mla_status mla_get_device_error(int32_t *code, void *stream) {
    if (!code) return MLA_ERR_INVALID_ARG;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return MLA_ERR_CUDA;
    int32_t v = 0;
    if (cudaMemcpyFromSymbol(&v, mla::g_device_error, sizeof(v)) != cudaSuccess) return MLA_ERR_CUDA;
    const int32_t zero = 0;
    if (cudaMemcpyToSymbol(mla::g_device_error, &zero, sizeof(zero)) != cudaSuccess) return MLA_ERR_CUDA;
    *code = v;
    return MLA_OK;
}

}  // extern "C"

namespace {
// Scratch for mla_decode_latent_noalloc: the partial results of the split-KV
// step live here instead of in a caller workspace. One copy per device.
static __device__ __align__(256) uint8_t g_noalloc_scratch[MLA_NOALLOC_SCRATCH_BYTES];

struct NoallocState {
    std::once_flag once;
    void *ptr = nullptr;
    mla_status status = MLA_OK;
};
NoallocState g_noalloc[kMaxDevices];

// Device address of this device's scratch array, looked up once per device
// with that device current.
mla_status noalloc_scratch(void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MLA_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return MLA_ERR_UNSUPPORTED;
    NoallocState &st = g_noalloc[dev];
    std::call_once(st.once, [&] {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p)
            st.status = MLA_ERR_CUDA;
        else
            st.ptr = p;
    });
    *out = st.ptr;
    return st.status;
}
}  // namespace

extern "C" {

mla_status mla_decode_latent_noalloc(const mla_dims *dims, const void *q, const mla_pool *ckv,
                                     const mla_pool *kr, int32_t num_pages,
                                     const int32_t *block_table, int32_t max_pages_per_seq,
                                     const int32_t *seq_lens, int32_t batch, int32_t num_parts,
                                     void *o_lat, float *lse_out, void *stream) {
    mla_status st = check_dims(dims, true);
    if (st != MLA_OK) return st;
    if (batch < 0 || num_parts <= 0) return MLA_ERR_INVALID_ARG;
    if (batch == 0) return MLA_OK;
    const size_t need = mla_decode_workspace_bytes(dims, batch, num_parts);
    if (need == 0 || need > MLA_NOALLOC_SCRATCH_BYTES) return MLA_ERR_INVALID_ARG;
    // the combine's own output checks, before the decode is launched
    if (!o_lat || !aligned(o_lat, 16) || (lse_out && !aligned(lse_out, 4)))
        return MLA_ERR_INVALID_ARG;
    if ((st = device_ready()) != MLA_OK) return st;
    void *scratch = nullptr;
    if ((st = noalloc_scratch(&scratch)) != MLA_OK) return st;
    st = mla_decode_splitkv(dims, q, ckv, kr, num_pages, block_table, max_pages_per_seq, seq_lens,
                            batch, num_parts, scratch, MLA_NOALLOC_SCRATCH_BYTES, stream);
    if (st != MLA_OK) return st;
    return mla_combine(dims, scratch, MLA_NOALLOC_SCRATCH_BYTES, seq_lens, max_pages_per_seq, batch,
                       num_parts, o_lat, lse_out, stream);
}

mla_status mla_combine_absorb_out(const mla_dims *dims, const void *workspace,
                                  size_t workspace_bytes, const int32_t *seq_lens,
                                  int32_t max_pages_per_seq, int32_t batch, int32_t num_parts,
                                  const void *w_uv, void *out, float *lse_out, void *stream) {
    mla_status st = check_dims(dims, true);
    if (st != MLA_OK) return st;
    if (batch < 0 || num_parts <= 0 || max_pages_per_seq <= 0) return MLA_ERR_INVALID_ARG;
    if (num_parts >= mla::kCoMaxSlots) return MLA_ERR_UNSUPPORTED;   // slots per sequence <= num_parts + 1
    const int32_t dc = dims->d_latent;
    if (dims->d_v > 128 || !(dc == 64 || dc == 128 || (dc % 128 == 0 && dc <= 1024)))
        return MLA_ERR_UNSUPPORTED;
    if (batch == 0) return MLA_OK;
    if (!workspace || !seq_lens || !w_uv || !out) return MLA_ERR_INVALID_ARG;
    if (!aligned(workspace, 256) || !aligned(w_uv, 16) || !aligned(out, 16) || !aligned(seq_lens, 4) ||
        (lse_out && !aligned(lse_out, 4)))
        return MLA_ERR_INVALID_ARG;
    if (workspace_bytes < mla_decode_workspace_bytes(dims, batch, num_parts)) return MLA_ERR_INVALID_ARG;
    if ((st = device_ready()) != MLA_OK) return st;
    const int64_t R = static_cast<int64_t>(dims->n_q) * dims->num_heads;
    const int64_t slots = static_cast<int64_t>(batch) + num_parts;
    const int64_t T64 = static_cast<int64_t>(batch) * dims->n_q;
    if (T64 > (int64_t(1) << 30)) return MLA_ERR_UNSUPPORTED;
    const int32_t T = static_cast<int32_t>(T64);
    const int32_t KS = dc >= 256 ? dc / 128 : 1;
    const int32_t KC = dc / KS;
    // Tokens per CTA: 16 (the smallest MMA N, the most CTAs; W_UV re-reads hit L2)
    // while the grid fits in one wave of five CTAs per SM; a larger one takes 32
    // (half the CTAs and waves, each W_UV slice read half as often).
    const int32_t NT =
        (static_cast<int64_t>(dims->num_heads) * KS * ((T + 15) / 16) > 5 * static_cast<int64_t>(device_sms()))
            ? 32
            : 16;
    CUtensorMap mw;
    if ((st = map_3d(&mw, w_uv, dims->d_v, dc, dims->num_heads, uint64_t(dims->d_v) * 2,
                     uint64_t(dc) * dims->d_v * 2, 64, 64, 1)) != MLA_OK)
        return st;
    mla::CombineOutArgs a;
    a.o_part = static_cast<const float *>(workspace);
    a.lse_part = reinterpret_cast<const float *>(static_cast<const uint8_t *>(workspace) +
                                                 round_up(slots * R * dc * 4, 256));
    a.seq_lens = seq_lens;
    a.out = static_cast<__nv_bfloat16 *>(out);
    a.lse_out = lse_out;
    a.timeout_ns = kDefaultTimeoutNs;
    a.batch = batch;
    a.max_pages = max_pages_per_seq;
    a.n_q = dims->n_q;
    a.H = dims->num_heads;
    a.rows = static_cast<int32_t>(R);
    a.d_c = dc;
    a.d_v = dims->d_v;
    a.tile_tokens = tile_tokens(variant_of(dims));
    a.num_parts = num_parts;
    a.T = T;
    a.NT = NT;
    a.KS = KS;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(dims->num_heads * KS), static_cast<unsigned>((T + NT - 1) / NT));
    cfg.blockDim = dim3(128);
    a.max_slots = num_parts + 1;   // < kCoMaxSlots + 1 (checked above)
    static_assert(32 * 128 * 4 <= 16384, "the partial D tile fits in one K block of W_UV rows");
    // Five CTAs fit on an SM: a grid larger than one wave at four per SM takes five
    // (fewer waves); one that fits is kept at four, spread over more SMs (the merge
    // is bound by each SM's load bandwidth), by requesting more than a fifth of
    // the SM's shared memory.
    uint32_t smem = mla::co_smem_bytes(KC, NT, a.max_slots);
    const int64_t grid = static_cast<int64_t>(dims->num_heads) * KS * ((T + NT - 1) / NT);
    if (grid <= 4 * static_cast<int64_t>(device_sms())) smem = std::max(smem, mla::kCoFourPerSmSmem);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = static_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(KS);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // as launch_pdl
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    if (cudaLaunchKernelEx(&cfg, mla::combine_out_kernel, mw, a) != cudaSuccess) return MLA_ERR_CUDA;
    return launch_status();
}

mla_status mla_debug_gather(const mla_pool *pool, int32_t width, int32_t num_pages,
                            const int32_t *block_table, int32_t max_pages_per_seq,
                            const int32_t *seq_lens, int32_t batch, int32_t max_len, void *out,
                            void *stream) {
    if (width < 8 || width > kGatherMaxWidth || (width % 8) || (width > 64 && (width % 64)))
        return MLA_ERR_INVALID_ARG;
    if (num_pages <= 0 || max_pages_per_seq <= 0 || batch < 0 || max_len <= 0) return MLA_ERR_INVALID_ARG;
    if (!block_table || !seq_lens || !out || !aligned(out, 16) || !aligned(block_table, 4) ||
        !aligned(seq_lens, 4))
        return MLA_ERR_INVALID_ARG;
    mla_status st = check_pool(pool, width);
    if (st != MLA_OK) return st;
    if ((st = device_ready()) != MLA_OK) return st;
    if (batch == 0) return MLA_OK;
    const uint32_t box_ch = static_cast<uint32_t>(width < 64 ? width : 64);
    CUtensorMap m;
    if ((st = pool_map(&m, pool, width, num_pages, box_ch, 64, CU_TENSOR_MAP_SWIZZLE_NONE)) != MLA_OK)
        return st;
    mla::GatherArgs a;
    a.block_table = block_table;
    a.seq_lens = seq_lens;
    a.out = static_cast<__nv_bfloat16 *>(out);
    a.timeout_ns = kDefaultTimeoutNs;
    a.batch = batch;
    a.max_pages = max_pages_per_seq;
    a.num_pages = num_pages;
    a.width = width;
    a.box_ch = static_cast<int32_t>(box_ch);
    a.max_len = max_len;
    dim3 grid(batch, max_pages_per_seq);
    mla::gather_kernel<<<grid, 128, 64 * width * 2, static_cast<cudaStream_t>(stream)>>>(m, a);
    return launch_status();
}

mla_status mla_debug_wait_timeout(int64_t timeout_ns, void *stream) {
    if (timeout_ns <= 0) return MLA_ERR_INVALID_ARG;
    mla_status st = device_ready();
    if (st != MLA_OK) return st;
    mla::wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(timeout_ns);
    return launch_status();
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Prefill through the decompress branch
// ---------------------------------------------------------------------------
namespace {

constexpr int32_t kDecompressHeadsPerCta = 8;

// The one compiled prefill specialisation: DeepSeek-V2/V3 dims.
mla_status check_prefill_dims(const mla_dims *d) {
    mla_status st = check_dims(d, false);
    if (st != MLA_OK) return st;
    if (d->d_latent != 512 || d->d_rope != 64 || d->d_nope != 128 || d->d_v != 128 ||
        d->page_size != 64)
        return MLA_ERR_UNSUPPORTED;
    return MLA_OK;
}

int64_t prefill_l_pad(int32_t max_pages) { return round_up(static_cast<int64_t>(max_pages) * 64, 128); }

int64_t prefill_half_bytes(const mla_dims *d, int32_t batch, int32_t max_pages) {
    return round_up(static_cast<int64_t>(batch) * d->num_heads * prefill_l_pad(max_pages) * 128 * 2,
                    256);
}

}  // namespace

extern "C" {

size_t mla_prefill_workspace_bytes(const mla_dims *dims, int32_t batch, int32_t max_pages_per_seq) {
    if (check_prefill_dims(dims) != MLA_OK || batch < 0 || max_pages_per_seq <= 0) return 0;
    return static_cast<size_t>(2 * prefill_half_bytes(dims, batch, max_pages_per_seq));
}

}  // extern "C"

namespace {

// Shared by the bf16 and E4M3 cache forms: ckv (bf16) or ckv8 + scales (E4M3).
mla_status decompress_common(const mla_dims *dims, const mla_pool *ckv, const mla_pool *ckv8,
                             const float *scales, int32_t num_pages, const int32_t *block_table,
                             int32_t max_pages_per_seq, const int32_t *seq_lens, int32_t batch,
                             const void *w_uk, const void *w_uv, void *workspace,
                             size_t workspace_bytes, void *stream) {
    mla_status st = check_prefill_dims(dims);
    if (st != MLA_OK) return st;
    if (batch < 0 || max_pages_per_seq <= 0 || num_pages <= 0) return MLA_ERR_INVALID_ARG;
    if (batch == 0) return MLA_OK;
    if (!block_table || !seq_lens || !w_uk || !w_uv || !workspace) return MLA_ERR_INVALID_ARG;
    if (!aligned(block_table, 4) || !aligned(seq_lens, 4) || !aligned(w_uk, 16) ||
        !aligned(w_uv, 16) || !aligned(workspace, 256))
        return MLA_ERR_INVALID_ARG;
    const bool fp8 = ckv8 != nullptr;
    if (fp8) {
        if (!ckv8->base || !scales || !aligned(ckv8->base, 16) || !aligned(scales, 4) ||
            ckv8->token_stride < dims->d_latent || ckv8->page_stride < 64 * ckv8->token_stride ||
            (ckv8->token_stride % 16) || (ckv8->page_stride % 16))
            return MLA_ERR_INVALID_ARG;
    } else if ((st = check_pool(ckv, dims->d_latent)) != MLA_OK) {
        return st;
    }
    if (workspace_bytes < mla_prefill_workspace_bytes(dims, batch, max_pages_per_seq))
        return MLA_ERR_INVALID_ARG;
    const int64_t l_pad = prefill_l_pad(max_pages_per_seq);
    const int64_t tiles = l_pad / mla::dkv::TOK;
    if (2 * static_cast<int64_t>(batch) * ((tiles + 1) / 2) > (int64_t(1) << 31) - 1 ||
        l_pad > (int64_t(1) << 30))
        return MLA_ERR_UNSUPPORTED;
    if ((st = device_ready()) != MLA_OK) return st;
    const int32_t H = dims->num_heads;
    CUtensorMap mc, mk, mv;
    // W_UK [H, d_n, d_c]: box [64 d x 64 c];  W_UV [H, d_c, d_v]: box [64 c x 64 e] (each CTA
    // of a pair loads its half of a chunk)
    if ((st = map_3d(&mk, w_uk, 512, 128, H, 512 * 2, uint64_t(128) * 512 * 2, 64, 64, 1)) != MLA_OK)
        return st;
    if ((st = map_3d(&mv, w_uv, 128, 512, H, 128 * 2, uint64_t(512) * 128 * 2, 64, 64, 1)) != MLA_OK)
        return st;
    if (fp8) {
        mc = mk;   // unused by the E4M3 form
    } else if ((st = pool_map(&mc, ckv, 512, num_pages, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B)) !=
               MLA_OK) {
        return st;
    }
    mla::DecompressArgs a;
    a.ckv8 = fp8 ? static_cast<const uint8_t *>(ckv8->base) : nullptr;
    a.scales = scales;
    a.ckv8_page_stride = fp8 ? ckv8->page_stride : 0;
    a.ckv8_token_stride = fp8 ? ckv8->token_stride : 0;
    a.block_table = block_table;
    a.seq_lens = seq_lens;
    a.k_nope = static_cast<__nv_bfloat16 *>(workspace);
    a.v = reinterpret_cast<__nv_bfloat16 *>(static_cast<uint8_t *>(workspace) +
                                            prefill_half_bytes(dims, batch, max_pages_per_seq));
    a.timeout_ns = kDefaultTimeoutNs;
    a.batch = batch;
    a.heads = H;
    a.max_pages = max_pages_per_seq;
    a.num_pages = num_pages;
    a.l_pad = static_cast<int32_t>(l_pad);
    a.pairs_per_seq = static_cast<int32_t>((tiles + 1) / 2);
    a.heads_per_cta = std::min(kDecompressHeadsPerCta, H);
    dim3 grid(static_cast<unsigned>(2 * batch * ((tiles + 1) / 2)),   // CTA pairs (clusters of 2)
              static_cast<unsigned>((H + a.heads_per_cta - 1) / a.heads_per_cta));
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (fp8)
        mla::decompress_kernel<true><<<grid, mla::dkv::THREADS, mla::dkv::SMEM_BYTES, s>>>(mc, mk, mv, a);
    else
        mla::decompress_kernel<false><<<grid, mla::dkv::THREADS, mla::dkv::SMEM_BYTES, s>>>(mc, mk, mv, a);
    return launch_status();
}

}  // namespace

extern "C" {

mla_status mla_decompress_kv(const mla_dims *dims, const mla_pool *ckv, int32_t num_pages,
                             const int32_t *block_table, int32_t max_pages_per_seq,
                             const int32_t *seq_lens, int32_t batch, const void *w_uk,
                             const void *w_uv, void *workspace, size_t workspace_bytes,
                             void *stream) {
    if (!ckv) return MLA_ERR_INVALID_ARG;
    return decompress_common(dims, ckv, nullptr, nullptr, num_pages, block_table,
                             max_pages_per_seq, seq_lens, batch, w_uk, w_uv, workspace,
                             workspace_bytes, stream);
}

mla_status mla_decompress_kv_fp8(const mla_dims *dims, const mla_pool *ckv8, const float *scales,
                                 int32_t num_pages, const int32_t *block_table,
                                 int32_t max_pages_per_seq, const int32_t *seq_lens, int32_t batch,
                                 const void *w_uk, const void *w_uv, void *workspace,
                                 size_t workspace_bytes, void *stream) {
    if (!ckv8) return MLA_ERR_INVALID_ARG;
    return decompress_common(dims, nullptr, ckv8, scales, num_pages, block_table,
                             max_pages_per_seq, seq_lens, batch, w_uk, w_uv, workspace,
                             workspace_bytes, stream);
}

}  // extern "C"

namespace {

// Every argument check of mla_prefill_attention (host only, nothing launched).
mla_status check_prefill_attention(const mla_dims *dims, const void *q_c, const void *q_r,
                                   const mla_pool *kr, int32_t num_pages,
                                   const int32_t *block_table, int32_t max_pages_per_seq,
                                   const int32_t *seq_lens, int32_t batch, const void *workspace,
                                   size_t workspace_bytes, const void *out, const float *lse) {
    mla_status st = check_prefill_dims(dims);
    if (st != MLA_OK) return st;
    if (batch < 0 || max_pages_per_seq <= 0 || num_pages <= 0) return MLA_ERR_INVALID_ARG;
    if (batch == 0) return MLA_OK;
    if (!q_c || !q_r || !block_table || !seq_lens || !workspace || !out) return MLA_ERR_INVALID_ARG;
    if (!aligned(q_c, 16) || !aligned(q_r, 16) || !aligned(block_table, 4) ||
        !aligned(seq_lens, 4) || !aligned(workspace, 256) || !aligned(out, 16) ||
        (lse && !aligned(lse, 4)))
        return MLA_ERR_INVALID_ARG;
    if ((st = check_pool(kr, dims->d_rope)) != MLA_OK) return st;
    if (workspace_bytes < mla_prefill_workspace_bytes(dims, batch, max_pages_per_seq))
        return MLA_ERR_INVALID_ARG;
    const int64_t M = dims->n_q, H = dims->num_heads;
    const int64_t q_blocks = (M + mla::pfa::ROWS - 1) / mla::pfa::ROWS;
    if (batch > 65535 || H > 65535 || q_blocks > (int64_t(1) << 31) - 1 ||
        static_cast<int64_t>(batch) * M > (int64_t(1) << 31) - 1)
        return MLA_ERR_UNSUPPORTED;
    return MLA_OK;
}

}  // namespace

extern "C" {

mla_status mla_prefill_attention(const mla_dims *dims, const void *q_c, const void *q_r,
                                 const mla_pool *kr, int32_t num_pages, const int32_t *block_table,
                                 int32_t max_pages_per_seq, const int32_t *seq_lens, int32_t batch,
                                 const void *workspace, size_t workspace_bytes, void *out,
                                 float *lse, void *stream) {
    mla_status st = check_prefill_attention(dims, q_c, q_r, kr, num_pages, block_table,
                                            max_pages_per_seq, seq_lens, batch, workspace,
                                            workspace_bytes, out, lse);
    if (st != MLA_OK || batch == 0) return st;
    const int64_t M = dims->n_q, H = dims->num_heads;
    const int64_t q_blocks = (M + mla::pfa::ROWS - 1) / mla::pfa::ROWS;
    if ((st = device_ready()) != MLA_OK) return st;
    const int64_t l_pad = prefill_l_pad(max_pages_per_seq);
    const uint64_t BM = static_cast<uint64_t>(batch) * M, BH = static_cast<uint64_t>(batch) * H;
    CUtensorMap mqc, mqr, mk, mv, mkr;
    if ((st = map_3d(&mqc, q_c, 128, H, BM, 128 * 2, uint64_t(H) * 128 * 2, 64, 1, 128)) != MLA_OK)
        return st;
    if ((st = map_3d(&mqr, q_r, 64, H, BM, 64 * 2, uint64_t(H) * 64 * 2, 64, 1, 128)) != MLA_OK)
        return st;
    const uint8_t *ws = static_cast<const uint8_t *>(workspace);
    if ((st = map_3d(&mk, ws, 128, l_pad, BH, 128 * 2, uint64_t(l_pad) * 128 * 2, 64, 128, 1)) !=
        MLA_OK)
        return st;
    if ((st = map_3d(&mv, ws + prefill_half_bytes(dims, batch, max_pages_per_seq), 128, l_pad, BH,
                     128 * 2, uint64_t(l_pad) * 128 * 2, 64, 128, 1)) != MLA_OK)
        return st;
    if ((st = pool_map(&mkr, kr, 64, num_pages, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B)) != MLA_OK)
        return st;
    mla::PrefillArgs a;
    a.block_table = block_table;
    a.seq_lens = seq_lens;
    a.out = static_cast<__nv_bfloat16 *>(out);
    a.lse = lse;
    a.timeout_ns = kDefaultTimeoutNs;
    a.batch = batch;
    a.heads = static_cast<int32_t>(H);
    a.n_q = static_cast<int32_t>(M);
    a.max_pages = max_pages_per_seq;
    a.num_pages = num_pages;
    a.l_pad = static_cast<int32_t>(l_pad);
    a.q_blocks = static_cast<int32_t>(q_blocks);
    a.scale = scale_of(dims);
    a.scale_log2 = a.scale * 1.4426950408889634f;
    dim3 grid(static_cast<unsigned>(q_blocks), static_cast<unsigned>(H), static_cast<unsigned>(batch));
    mla::prefill_attn_kernel<<<grid, mla::pfa::THREADS, mla::pfa::SMEM_BYTES,
                               static_cast<cudaStream_t>(stream)>>>(mqc, mqr, mk, mv, mkr, a);
    return launch_status();
}

mla_status mla_prefill(const mla_dims *dims, const void *q_c, const void *q_r, const mla_pool *ckv,
                       const mla_pool *kr, int32_t num_pages, const int32_t *block_table,
                       int32_t max_pages_per_seq, const int32_t *seq_lens, int32_t batch,
                       const void *w_uk, const void *w_uv, void *workspace,
                       size_t workspace_bytes, void *out, float *lse, void *stream) {
    // both steps' arguments are checked before the first launch
    mla_status st = check_prefill_attention(dims, q_c, q_r, kr, num_pages, block_table,
                                            max_pages_per_seq, seq_lens, batch, workspace,
                                            workspace_bytes, out, lse);
    if (st != MLA_OK || batch == 0) return st;
    if ((st = mla_decompress_kv(dims, ckv, num_pages, block_table, max_pages_per_seq, seq_lens,
                                batch, w_uk, w_uv, workspace, workspace_bytes, stream)) != MLA_OK)
        return st;
    return mla_prefill_attention(dims, q_c, q_r, kr, num_pages, block_table, max_pages_per_seq,
                                 seq_lens, batch, workspace, workspace_bytes, out, lse, stream);
}

}  // extern "C"


namespace {

mla_status append_common(const mla_dims *dims, const void *ckv_new, const void *kr_new,
                         const int32_t *seq_ids, const int32_t *positions, int32_t num_tokens,
                         float rope_theta, const mla_pool *ckv, const mla_pool *ckv8, float *scales,
                         const mla_pool *kr, int32_t num_pages, const int32_t *block_table,
                         int32_t max_pages_per_seq, int32_t batch, void *stream) {
    mla_status st = check_dims(dims, false);
    if (st != MLA_OK) return st;
    if (dims->page_size != 64 || (dims->d_rope % 2)) return MLA_ERR_UNSUPPORTED;
    if (num_tokens < 0 || batch < 0 || max_pages_per_seq <= 0 || num_pages <= 0 ||
        !std::isfinite(rope_theta))
        return MLA_ERR_INVALID_ARG;
    if (num_tokens == 0) return MLA_OK;
    if (!ckv_new || !kr_new || !seq_ids || !positions || !block_table) return MLA_ERR_INVALID_ARG;
    if (!aligned(ckv_new, 16) || !aligned(kr_new, 2) || !aligned(seq_ids, 4) ||
        !aligned(positions, 4) || !aligned(block_table, 4))
        return MLA_ERR_INVALID_ARG;
    const bool fp8 = ckv8 != nullptr;
    if (fp8) {
        if (dims->d_latent % 16) return MLA_ERR_UNSUPPORTED;
        if (!ckv8->base || !scales || !aligned(ckv8->base, 16) || !aligned(scales, 4) ||
            ckv8->token_stride < dims->d_latent || ckv8->page_stride < 64 * ckv8->token_stride ||
            (ckv8->token_stride % 16) || (ckv8->page_stride % 16))
            return MLA_ERR_INVALID_ARG;
    } else if ((st = check_pool(ckv, dims->d_latent)) != MLA_OK) {
        return st;
    }
    if (!kr || !kr->base || !aligned(kr->base, 2) || kr->token_stride < dims->d_rope ||
        kr->page_stride < kr->token_stride)
        return MLA_ERR_INVALID_ARG;
    if ((st = device_ready()) != MLA_OK) return st;
    mla::AppendArgs a;
    a.ckv_new = static_cast<const __nv_bfloat16 *>(ckv_new);
    a.kr_new = static_cast<const __nv_bfloat16 *>(kr_new);
    a.seq_ids = seq_ids;
    a.positions = positions;
    a.block_table = block_table;
    a.ckv = fp8 ? nullptr : static_cast<__nv_bfloat16 *>(const_cast<void *>(ckv->base));
    a.ckv8 = fp8 ? static_cast<uint8_t *>(const_cast<void *>(ckv8->base)) : nullptr;
    a.scales = scales;
    a.kr = static_cast<__nv_bfloat16 *>(const_cast<void *>(kr->base));
    a.ckv_page_stride = fp8 ? ckv8->page_stride : ckv->page_stride;
    a.ckv_token_stride = fp8 ? ckv8->token_stride : ckv->token_stride;
    a.kr_page_stride = kr->page_stride;
    a.kr_token_stride = kr->token_stride;
    a.rotate = rope_theta > 0.f ? 1 : 0;
    a.log_theta = rope_theta > 0.f ? std::log(static_cast<double>(rope_theta)) : 0.0;
    a.T = num_tokens;
    a.d_c = dims->d_latent;
    a.d_r = dims->d_rope;
    a.batch = batch;
    a.max_pages = max_pages_per_seq;
    a.num_pages = num_pages;
    mla::append_kv_kernel<<<(num_tokens + 7) / 8, 256, 0, static_cast<cudaStream_t>(stream)>>>(a);
    return launch_status();
}

}  // namespace

extern "C" {

mla_status mla_append_kv(const mla_dims *dims, const void *ckv_new, const void *kr_new,
                         const int32_t *seq_ids, const int32_t *positions, int32_t num_tokens,
                         float rope_theta, const mla_pool *ckv, const mla_pool *kr,
                         int32_t num_pages, const int32_t *block_table, int32_t max_pages_per_seq,
                         int32_t batch, void *stream) {
    if (!ckv) return MLA_ERR_INVALID_ARG;
    return append_common(dims, ckv_new, kr_new, seq_ids, positions, num_tokens, rope_theta, ckv,
                         nullptr, nullptr, kr, num_pages, block_table, max_pages_per_seq, batch,
                         stream);
}

mla_status mla_append_kv_fp8(const mla_dims *dims, const void *ckv_new, const void *kr_new,
                             const int32_t *seq_ids, const int32_t *positions, int32_t num_tokens,
                             float rope_theta, const mla_pool *ckv8, float *scales,
                             const mla_pool *kr, int32_t num_pages, const int32_t *block_table,
                             int32_t max_pages_per_seq, int32_t batch, void *stream) {
    if (!ckv8) return MLA_ERR_INVALID_ARG;
    return append_common(dims, ckv_new, kr_new, seq_ids, positions, num_tokens, rope_theta,
                         nullptr, ckv8, scales, kr, num_pages, block_table, max_pages_per_seq,
                         batch, stream);
}

mla_status mla_gather_dequant_fp8(const mla_pool *ckv8, const float *scales, int32_t width,
                                  int32_t num_pages, const int32_t *block_table,
                                  int32_t max_pages_per_seq, const int32_t *seq_lens,
                                  int32_t batch, int32_t max_len, void *out, void *stream) {
    if (width < 16 || width > 4096 || (width % 16)) return MLA_ERR_UNSUPPORTED;
    if (!ckv8 || !ckv8->base || !scales || !block_table || !seq_lens || !out)
        return MLA_ERR_INVALID_ARG;
    if (batch < 0 || max_len < 0 || max_pages_per_seq <= 0 || num_pages <= 0)
        return MLA_ERR_INVALID_ARG;
    if (!aligned(ckv8->base, 16) || !aligned(scales, 4) || !aligned(block_table, 4) ||
        !aligned(seq_lens, 4) || !aligned(out, 16) || ckv8->token_stride < width ||
        ckv8->page_stride < 64 * ckv8->token_stride || (ckv8->token_stride % 16) ||
        (ckv8->page_stride % 16))
        return MLA_ERR_INVALID_ARG;
    if (batch == 0 || max_len == 0) return MLA_OK;
    const int64_t rows = static_cast<int64_t>(batch) * max_len;
    if ((rows + 7) / 8 > (int64_t(1) << 31) - 1) return MLA_ERR_UNSUPPORTED;
    mla_status st = device_ready();
    if (st != MLA_OK) return st;
    mla::GatherFp8Args a;
    a.ckv8 = static_cast<const uint8_t *>(ckv8->base);
    a.scales = scales;
    a.block_table = block_table;
    a.seq_lens = seq_lens;
    a.out = static_cast<__nv_bfloat16 *>(out);
    a.page_stride = ckv8->page_stride;
    a.token_stride = ckv8->token_stride;
    a.width = width;
    a.num_pages = num_pages;
    a.max_pages = max_pages_per_seq;
    a.batch = batch;
    a.max_len = max_len;
    mla::gather_dequant_fp8_kernel<<<static_cast<unsigned>((rows + 7) / 8), 256, 0,
                                     static_cast<cudaStream_t>(stream)>>>(a);
    return launch_status();
}

}  // extern "C"
