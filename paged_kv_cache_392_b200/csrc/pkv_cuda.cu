// Host side of libpkv's CUDA path: argument validation, kernel selection and launches for
// paged_attn_decode, kv_write and kv_copy_blocks, plus the device fault word.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <climits>
#include <cmath>
#include <mutex>

#include "attn_decode.cuh"
#include "attn_decode_fp8.cuh"
#include "attn_decode_tc.cuh"
#include "kv_ops.cuh"
#include "read_probe.cuh"
#include "pkv_internal.h"

namespace {

using pkv::fail;

constexpr int kWarps = PKV_DECODE_WARPS;    // consumer warps per decode CTA
constexpr int kStages = PKV_DECODE_STAGES;  // shared-memory stages per warp (K+V block each)
constexpr int kMaxDevices = 64;
constexpr int kDefaultPartitionTokens = pkv::kDefaultPartitionTokens;

int elem_size(int32_t dtype) {
    return dtype == PKV_F32 ? 4
           : (dtype == PKV_F16 || dtype == PKV_BF16) ? 2
           : dtype == PKV_FP8_E4M3 ? 1
           : 0;
}

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// log2 of the tokens per physical block (16 or 32; checked by check_pool_desc).
int32_t block_shift(const pkv_attn_desc *d) { return d->block_size == 32 ? 5 : 4; }

// 16-token sub-blocks the longest admissible sequence spans.
int64_t sub_blocks_per_seq(const pkv_attn_desc *d) {
    return (int64_t)d->max_blocks_per_seq * (d->block_size / pkv::kBlock);
}

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Checks shared by every entry point that touches the pools.
pkv_status check_pool_desc(const pkv_attn_desc *d, const char *fn) {
    if (!d) return fail(PKV_ERR_INVALID, "%s: desc is NULL", fn);
    if (!elem_size(d->dtype)) return fail(PKV_ERR_INVALID, "%s: unknown dtype %d", fn, d->dtype);
    if (d->block_size != 16 && d->block_size != 32)
        return fail(PKV_ERR_UNSUPPORTED, "%s: block_size %d (16 or 32)", fn, d->block_size);
    if (d->head_dim != 64 && d->head_dim != 128)
        return fail(PKV_ERR_UNSUPPORTED, "%s: head_dim %d (64 or 128)", fn, d->head_dim);
    if (d->num_kv_heads < 1) return fail(PKV_ERR_INVALID, "%s: num_kv_heads < 1", fn);
    if (d->num_blocks < 1) return fail(PKV_ERR_INVALID, "%s: num_blocks < 1", fn);
    if ((int64_t)d->num_blocks * d->block_size > INT64_MAX / 2)
        return fail(PKV_ERR_INVALID, "%s: num_blocks too large", fn);
    return PKV_OK;
}

struct Split {
    int32_t part_blocks;
    int32_t pmax;
};

pkv_status check_attn_desc(const pkv_attn_desc *d, const char *fn, Split *sp) {
    pkv_status st = check_pool_desc(d, fn);
    if (st) return st;
    if (d->dtype == PKV_FP8_E4M3)
        return fail(PKV_ERR_INVALID, "%s: desc->dtype is the q/out type (f32, f16, bf16)", fn);
    if (d->num_seqs < 0) return fail(PKV_ERR_INVALID, "%s: num_seqs < 0", fn);
    if (d->num_q_heads < 1 || d->num_q_heads % d->num_kv_heads)
        return fail(PKV_ERR_INVALID, "%s: num_q_heads %d not a multiple of num_kv_heads %d", fn,
                    d->num_q_heads, d->num_kv_heads);
    const int g = d->num_q_heads / d->num_kv_heads;
    if (g != 1 && g != 2 && g != 4 && g != 8)
        return fail(PKV_ERR_UNSUPPORTED, "%s: query heads per kv head %d (1, 2, 4 or 8)", fn, g);
    if (d->dtype == PKV_F32 && d->head_dim == 128 && g == 8)
        return fail(PKV_ERR_UNSUPPORTED, "%s: fp32 with head_dim 128 and group 8", fn);
    if (d->max_blocks_per_seq < 1 || d->max_blocks_per_seq > INT_MAX / d->block_size)
        return fail(PKV_ERR_INVALID, "%s: max_blocks_per_seq %d", fn, d->max_blocks_per_seq);
    if (d->partition_tokens < 0 || d->partition_tokens % pkv::kBlock)
        return fail(PKV_ERR_INVALID, "%s: partition_tokens %d not a multiple of 16", fn,
                    d->partition_tokens);
    const int32_t pt = d->partition_tokens ? d->partition_tokens : kDefaultPartitionTokens;
    sp->part_blocks = pt / pkv::kBlock;  // partitions count 16-token sub-blocks
    sp->pmax = (sub_blocks_per_seq(d) + sp->part_blocks - 1) / sp->part_blocks;
    const int64_t grid = (int64_t)d->num_seqs * d->num_kv_heads * sp->pmax;
    if (grid > INT_MAX || (int64_t)d->num_seqs * d->num_q_heads > INT_MAX)
        return fail(PKV_ERR_INVALID, "%s: batch too large for one launch", fn);
    return PKV_OK;
}

size_t workspace_bytes(const pkv_attn_desc *d, const Split &sp) {
    if (sp.pmax <= 1) return 0;
    const size_t rows = (size_t)d->num_seqs * d->num_q_heads * sp.pmax;
    return round_up(rows * d->head_dim * sizeof(float), 256) + rows * 2 * sizeof(float);
}

pkv_status cuda_check(cudaError_t e, const char *fn, const char *what) {
    if (e == cudaSuccess) return PKV_OK;
    return fail(PKV_ERR_CUDA, "%s: %s: %s", fn, what, cudaGetErrorString(e));
}

// Opt each decode instantiation into its dynamic shared memory once per device.
template <typename Kernel>
pkv_status ensure_smem(Kernel kern, int bytes, std::atomic<bool> *done, const char *fn) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_check(e, fn, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return fail(PKV_ERR_CUDA, "%s: device %d", fn, dev);
    if (done[dev].load(std::memory_order_acquire)) return PKV_OK;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return cuda_check(e, fn, "cudaFuncSetAttribute");
    done[dev].store(true, std::memory_order_release);
    return PKV_OK;
}

// cuTensorMapEncodeTiled from the driver, looked up once through the runtime (no libcuda
// link dependency).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            f = nullptr;
        return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    }();
    return fn;
}

// 2-D view [rows = NB*H_kv*16][D] of a 16-bit pool, boxes of 16 rows x 64 columns (128 B)
// with the 128-byte swizzle.
pkv_status kv_tensor_map(CUtensorMap *m, const void *pool, int32_t dtype, int D, int64_t rows,
                         const char *fn) {
    auto enc = tensor_map_encoder();
    if (!enc) return fail(PKV_ERR_CUDA, "%s: cuTensorMapEncodeTiled unavailable", fn);
    const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)D * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)pkv::kBlock};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(m, dtype == PKV_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                          : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                     2, const_cast<void *>(pool), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
        return fail(PKV_ERR_CUDA, "%s: cuTensorMapEncodeTiled failed (%d)", fn, (int)r);
    return PKV_OK;
}

// The log-sum-exp reduce after a split decode: one warp per row when no row can have more
// than kReduceBatch partitions (pmax bounds them all), else kReduceWideWarps warps per row.
template <typename T, int D>
pkv_status launch_reduce_if_split(const pkv::DecodeParams &prm, cudaStream_t stream) {
    if (prm.pmax <= 1) return PKV_OK;
    const int64_t rows = (int64_t)prm.S * prm.Hq;
    const bool narrow = prm.pmax <= pkv::kReduceBatch;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(narrow ? (rows + 3) / 4 : rows));
    cfg.blockDim = dim3(narrow ? 128 : pkv::kReduceWideWarps * 32);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e =
        narrow ? cudaLaunchKernelEx(&cfg, pkv::lse_reduce_kernel<T, D, 1>, prm)
               : cudaLaunchKernelEx(&cfg, pkv::lse_reduce_kernel<T, D, pkv::kReduceWideWarps>, prm);
    return cuda_check(e, "paged_attn_decode", "reduce launch");
}

constexpr int kTcWarps = PKV_DECODE_TC_WARPS;
constexpr int kTcStages = PKV_DECODE_TC_STAGES;

// Tensor-core decode for 16-bit K/V: the paged pools, or (kContig) a contiguous cache.
template <typename T, int D, int G, bool kContig = false>
pkv_status launch_decode_tc(const pkv::DecodeParams &prm, int32_t dtype, cudaStream_t stream) {
    using Cfg = pkv::DecodeTcCfg<T, D, G, kTcWarps, kTcStages>;
    auto kern = kContig ? pkv::contiguous_attn_decode_tc_kernel<T, D, G, kTcWarps, kTcStages>
                        : pkv::paged_attn_decode_tc_kernel<T, D, G, kTcWarps, kTcStages>;
    static std::atomic<bool> done[kMaxDevices];
    pkv_status st = ensure_smem(kern, Cfg::SMEM, done, "paged_attn_decode");
    if (st) return st;
    const int64_t rows = kContig ? (int64_t)prm.S * prm.Hkv * prm.Lmax
                                 : ((int64_t)prm.NB * prm.Hkv) << prm.bshift;
    CUtensorMap tmk, tmv;
    st = kv_tensor_map(&tmk, prm.k_pool, dtype, D, rows, "paged_attn_decode");
    if (st) return st;
    st = kv_tensor_map(&tmv, prm.v_pool, dtype, D, rows, "paged_attn_decode");
    if (st) return st;
    const unsigned grid = (unsigned)((int64_t)prm.S * prm.Hkv * prm.pmax);
    kern<<<grid, kTcWarps * 32, Cfg::SMEM, stream>>>(tmk, tmv, prm);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_check(e, "paged_attn_decode", "decode launch");
    return launch_reduce_if_split<T, D>(prm, stream);
}

template <typename T, int D, int G>
pkv_status launch_decode(const pkv::DecodeParams &prm, cudaStream_t stream) {
    using Cfg = pkv::DecodeCfg<T, D, G, kWarps, kStages>;
    auto kern = pkv::paged_attn_decode_kernel<T, D, G, kWarps, kStages>;
    static std::atomic<bool> done[kMaxDevices];
    pkv_status st = ensure_smem(kern, Cfg::SMEM, done, "paged_attn_decode");
    if (st) return st;
    const unsigned grid = (unsigned)((int64_t)prm.S * prm.Hkv * prm.pmax);
    kern<<<grid, kWarps * 32, Cfg::SMEM, stream>>>(prm);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_check(e, "paged_attn_decode", "decode launch");
    return launch_reduce_if_split<T, D>(prm, stream);
}

// Whether the tensor-core kernel serves this call: 16-bit K/V whose 2-D TMA view fits int32
// row coordinates.  PKV_DECODE_FORCE_SIMT builds keep every call on the CUDA-core kernel.
bool use_tc(const pkv_attn_desc *d) {
#ifdef PKV_DECODE_FORCE_SIMT
    (void)d;
    return false;
#else
    return d->dtype != PKV_F32 &&
           (int64_t)d->num_blocks * d->num_kv_heads * d->block_size < ((int64_t)1 << 31);
#endif
}

template <typename T, int D, bool kContig = false>
pkv_status dispatch_group_tc(int g, const pkv::DecodeParams &prm, int32_t dtype,
                             cudaStream_t stream) {
    switch (g) {
    case 1: return launch_decode_tc<T, D, 1, kContig>(prm, dtype, stream);
    case 2: return launch_decode_tc<T, D, 2, kContig>(prm, dtype, stream);
    case 4: return launch_decode_tc<T, D, 4, kContig>(prm, dtype, stream);
    case 8: return launch_decode_tc<T, D, 8, kContig>(prm, dtype, stream);
    default: return fail(PKV_ERR_UNSUPPORTED, "paged_attn_decode: group %d", g);
    }
}

template <typename T, int D>
pkv_status dispatch_group(int g, const pkv::DecodeParams &prm, cudaStream_t stream) {
    switch (g) {
    case 1: return launch_decode<T, D, 1>(prm, stream);
    case 2: return launch_decode<T, D, 2>(prm, stream);
    case 4: return launch_decode<T, D, 4>(prm, stream);
    case 8:
        if constexpr (sizeof(T) == 4 && D == 128)
            return fail(PKV_ERR_UNSUPPORTED, "paged_attn_decode: fp32, D 128, group 8");
        else
            return launch_decode<T, D, 8>(prm, stream);
    default: return fail(PKV_ERR_UNSUPPORTED, "paged_attn_decode: group %d", g);
    }
}

template <typename T>
pkv_status dispatch_dim(int D, int g, const pkv::DecodeParams &prm, cudaStream_t stream) {
    if (D == 64) return dispatch_group<T, 64>(g, prm, stream);
    return dispatch_group<T, 128>(g, prm, stream);
}

int device_sm_count();

// Grid of a kv_write / kv_write_fp8 launch: one row of CTAs per tile of kTileTokens tokens
// (each CTA checks its tile's slots against the whole call), and as many slices of a tile's
// `items_per_token * tokens` items as keep about four CTAs per SM busy when there are few
// tiles (a decode step's write), down to one per tile for long writes, where every slice
// would repeat the tile's duplicate check.
pkv_status write_grid(int32_t tokens, int64_t items_per_token, dim3 *grid, const char *fn) {
    const int64_t tiles = (tokens + pkv::kTileTokens - 1) / pkv::kTileTokens;
    const int64_t tile_items = items_per_token * std::min<int64_t>(tokens, pkv::kTileTokens);
    if (tiles > INT_MAX || tile_items > INT_MAX / 2)
        return fail(PKV_ERR_INVALID, "%s: too many tokens or heads for one launch", fn);
    const int64_t sms = std::max(1, device_sm_count());
    const int64_t by_items = (tile_items + pkv::kWriteThreads - 1) / pkv::kWriteThreads;
    const int64_t by_sms = (4 * sms + tiles - 1) / tiles;
    const int64_t slices = std::max<int64_t>(1, std::min<int64_t>({by_items, by_sms, 65535}));
    *grid = dim3((unsigned)tiles, (unsigned)slices);
    return PKV_OK;
}

// Shared body of paged_attn_decode and kv_write_and_decode (k_new / v_new / slot_mapping
// NULL: no fused write).
pkv_status decode_impl(const pkv_attn_desc *desc, const void *q, const void *k_new,
                       const void *v_new, const int64_t *slot_mapping, const void *k_pool,
                       const void *v_pool, const int32_t *block_tables,
                       const int32_t *context_lens, float scale, void *out, void *workspace,
                       size_t workspace_bytes_given, void *stream, const char *fn) {
    Split sp;
    pkv_status st = check_attn_desc(desc, fn, &sp);
    if (st) return st;
    if (desc->num_seqs == 0) return PKV_OK;
    if (!q || !k_pool || !v_pool || !block_tables || !context_lens || !out)
        return fail(PKV_ERR_INVALID, "%s: NULL tensor pointer", fn);
    if (!aligned(q, 16) || !aligned(k_pool, 16) || !aligned(v_pool, 16) || !aligned(out, 16))
        return fail(PKV_ERR_INVALID, "%s: q, pools and out must be 16-byte aligned", fn);
    if (!aligned(block_tables, 4) || !aligned(context_lens, 4))
        return fail(PKV_ERR_INVALID, "%s: block_tables / context_lens misaligned", fn);
    if (!std::isfinite(scale)) return fail(PKV_ERR_INVALID, "%s: scale is not finite", fn);
    const size_t need = workspace_bytes(desc, sp);
    if (need) {
        if (!workspace || workspace_bytes_given < need)
            return fail(PKV_ERR_INVALID, "%s: workspace needs %zu bytes, got %zu", fn, need,
                        workspace ? workspace_bytes_given : (size_t)0);
        if (!aligned(workspace, 256))
            return fail(PKV_ERR_INVALID, "%s: workspace must be 256-byte aligned", fn);
    }
    pkv::DecodeParams prm;
    prm.q = q;
    prm.k_pool = k_pool;
    prm.v_pool = v_pool;
    prm.k_new = k_new;
    prm.v_new = v_new;
    prm.slot_mapping = slot_mapping;
    prm.block_tables = block_tables;
    prm.context_lens = context_lens;
    prm.out = out;
    const size_t rows = (size_t)desc->num_seqs * desc->num_q_heads * sp.pmax;
    prm.ws_o = need ? static_cast<float *>(workspace) : nullptr;
    prm.ws_ml = need ? reinterpret_cast<float *>(static_cast<char *>(workspace) +
                                                 round_up(rows * desc->head_dim * 4, 256))
                     : nullptr;
    prm.S = desc->num_seqs;
    prm.Hq = desc->num_q_heads;
    prm.Hkv = desc->num_kv_heads;
    prm.NB = desc->num_blocks;
    prm.maxB = desc->max_blocks_per_seq;
    prm.part_blocks = sp.part_blocks;
    prm.pmax = sp.pmax;
    prm.scale_log2 = scale * 1.4426950408889634f;
    prm.bshift = block_shift(desc);
    const int g = desc->num_q_heads / desc->num_kv_heads;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (use_tc(desc)) {
        if (desc->dtype == PKV_F16)
            return desc->head_dim == 64 ? dispatch_group_tc<__half, 64>(g, prm, PKV_F16, s)
                                        : dispatch_group_tc<__half, 128>(g, prm, PKV_F16, s);
        return desc->head_dim == 64
                   ? dispatch_group_tc<__nv_bfloat16, 64>(g, prm, PKV_BF16, s)
                   : dispatch_group_tc<__nv_bfloat16, 128>(g, prm, PKV_BF16, s);
    }
    switch (desc->dtype) {
    case PKV_F32: return dispatch_dim<float>(desc->head_dim, g, prm, s);
    case PKV_F16: return dispatch_dim<__half>(desc->head_dim, g, prm, s);
    default: return dispatch_dim<__nv_bfloat16>(desc->head_dim, g, prm, s);
    }
}

}  // namespace

extern "C" {

size_t pkv_attn_workspace_bytes(const pkv_attn_desc *desc) {
    pkv::clear_error();
    Split sp;
    if (check_attn_desc(desc, "pkv_attn_workspace_bytes", &sp)) return 0;
    return workspace_bytes(desc, sp);
}

pkv_status paged_attn_decode(const pkv_attn_desc *desc, const void *q, const void *k_pool,
                             const void *v_pool, const int32_t *block_tables,
                             const int32_t *context_lens, float scale, void *out,
                             void *workspace, size_t workspace_bytes_given, void *stream) {
    return decode_impl(desc, q, nullptr, nullptr, nullptr, k_pool, v_pool, block_tables,
                       context_lens, scale, out, workspace, workspace_bytes_given, stream,
                       "paged_attn_decode");
}

pkv_status kv_write_and_decode(const pkv_attn_desc *desc, const void *q, const void *k_new,
                               const void *v_new, const int64_t *slot_mapping, void *k_pool,
                               void *v_pool, const int32_t *block_tables,
                               const int32_t *context_lens, float scale, void *out,
                               void *workspace, size_t workspace_bytes_given, void *stream) {
    const char *fn = "kv_write_and_decode";
    if (desc && desc->dtype == PKV_FP8_E4M3)
        return fail(PKV_ERR_INVALID, "%s: FP8 pools are written by kv_write_fp8", fn);
    if (desc && desc->num_seqs > 0) {
        if (!k_new || !v_new || !slot_mapping)
            return fail(PKV_ERR_INVALID, "%s: NULL tensor pointer", fn);
        if (!aligned(k_new, 16) || !aligned(v_new, 16) || !aligned(slot_mapping, 8))
            return fail(PKV_ERR_INVALID, "%s: misaligned pointer", fn);
    }
    return decode_impl(desc, q, k_new, v_new, slot_mapping, k_pool, v_pool, block_tables,
                       context_lens, scale, out, workspace, workspace_bytes_given, stream, fn);
}

pkv_status kv_write(const pkv_attn_desc *desc, const void *k_new, const void *v_new,
                    const int64_t *slot_mapping, int32_t num_tokens, void *k_pool,
                    void *v_pool, void *stream) {
    const char *fn = "kv_write";
    pkv_status st = check_pool_desc(desc, fn);
    if (st) return st;
    if (desc->dtype == PKV_FP8_E4M3)
        return fail(PKV_ERR_INVALID, "%s: FP8 pools are written by kv_write_fp8", fn);
    if (num_tokens < 0) return fail(PKV_ERR_INVALID, "%s: num_tokens < 0", fn);
    if (num_tokens == 0) return PKV_OK;
    if (!k_new || !v_new || !slot_mapping || !k_pool || !v_pool)
        return fail(PKV_ERR_INVALID, "%s: NULL tensor pointer", fn);
    if (!aligned(k_new, 16) || !aligned(v_new, 16) || !aligned(k_pool, 16) ||
        !aligned(v_pool, 16) || !aligned(slot_mapping, 8))
        return fail(PKV_ERR_INVALID, "%s: misaligned pointer", fn);
    pkv::KvWriteParams prm;
    prm.k_new = static_cast<const uint4 *>(k_new);
    prm.v_new = static_cast<const uint4 *>(v_new);
    prm.slot_mapping = slot_mapping;
    prm.k_pool = static_cast<uint4 *>(k_pool);
    prm.v_pool = static_cast<uint4 *>(v_pool);
    prm.T = num_tokens;
    prm.Hkv = desc->num_kv_heads;
    prm.NB = desc->num_blocks;
    prm.vpr = desc->head_dim * elem_size(desc->dtype) / 16;
    prm.bshift = block_shift(desc);
    dim3 grid;
    st = write_grid(num_tokens, 2LL * prm.Hkv * prm.vpr, &grid, fn);
    if (st) return st;
    pkv::kv_write_kernel<<<grid, pkv::kWriteThreads, 0, static_cast<cudaStream_t>(stream)>>>(prm);
    return cuda_check(cudaGetLastError(), fn, "launch");
}

pkv_status kv_copy_blocks(const pkv_attn_desc *desc, const int32_t *src_dst_pairs,
                          int32_t num_pairs, void *k_pool, void *v_pool, void *stream) {
    const char *fn = "kv_copy_blocks";
    pkv_status st = check_pool_desc(desc, fn);
    if (st) return st;
    if (num_pairs < 0) return fail(PKV_ERR_INVALID, "%s: num_pairs < 0", fn);
    if (num_pairs == 0) return PKV_OK;
    if (!src_dst_pairs || !k_pool || !v_pool)
        return fail(PKV_ERR_INVALID, "%s: NULL pointer", fn);
    if (!aligned(k_pool, 16) || !aligned(v_pool, 16) || !aligned(src_dst_pairs, 4))
        return fail(PKV_ERR_INVALID, "%s: misaligned pointer", fn);
    if (num_pairs > INT_MAX / 2) return fail(PKV_ERR_INVALID, "%s: too many pairs", fn);
    pkv::KvCopyParams prm;
    prm.pairs = src_dst_pairs;
    prm.k_pool = static_cast<uint4 *>(k_pool);
    prm.v_pool = static_cast<uint4 *>(v_pool);
    prm.P = num_pairs;
    prm.NB = desc->num_blocks;
    prm.vpb = (int64_t)desc->num_kv_heads * desc->block_size * desc->head_dim *
              elem_size(desc->dtype) / 16;
    const int64_t slices = (prm.vpb + pkv::kCopyUnroll * 256 - 1) / (pkv::kCopyUnroll * 256);
    if (slices > 65535) return fail(PKV_ERR_UNSUPPORTED, "%s: block too large", fn);
    dim3 grid((unsigned)(2 * num_pairs), (unsigned)slices);
    pkv::kv_copy_blocks_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(prm);
    return cuda_check(cudaGetLastError(), fn, "launch");
}

pkv_status attn_decode_contiguous(const pkv_attn_desc *desc, const void *q, const void *k_cache,
                                  const void *v_cache, const int32_t *context_lens, float scale,
                                  void *out, void *workspace, size_t workspace_bytes_given,
                                  void *stream) {
    const char *fn = "attn_decode_contiguous";
    Split sp;
    pkv_status st = check_attn_desc(desc, fn, &sp);
    if (st) return st;
    if (desc->dtype != PKV_F16 && desc->dtype != PKV_BF16)
        return fail(PKV_ERR_UNSUPPORTED, "%s: 16-bit caches only (f16, bf16)", fn);
    const int64_t lmax = (int64_t)desc->max_blocks_per_seq * desc->block_size;
    if ((int64_t)desc->num_seqs * desc->num_kv_heads * lmax >= ((int64_t)1 << 31))
        return fail(PKV_ERR_UNSUPPORTED, "%s: cache too large for 32-bit TMA rows", fn);
    if (desc->num_seqs == 0) return PKV_OK;
    if (!q || !k_cache || !v_cache || !context_lens || !out)
        return fail(PKV_ERR_INVALID, "%s: NULL tensor pointer", fn);
    if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(out, 16) ||
        !aligned(context_lens, 4))
        return fail(PKV_ERR_INVALID, "%s: misaligned pointer", fn);
    if (!std::isfinite(scale)) return fail(PKV_ERR_INVALID, "%s: scale is not finite", fn);
    const size_t need = workspace_bytes(desc, sp);
    if (need) {
        if (!workspace || workspace_bytes_given < need)
            return fail(PKV_ERR_INVALID, "%s: workspace needs %zu bytes", fn, need);
        if (!aligned(workspace, 256))
            return fail(PKV_ERR_INVALID, "%s: workspace must be 256-byte aligned", fn);
    }
    pkv::DecodeParams prm;
    prm.q = q;
    prm.k_pool = k_cache;
    prm.v_pool = v_cache;
    prm.block_tables = nullptr;
    prm.context_lens = context_lens;
    prm.out = out;
    const size_t rows = (size_t)desc->num_seqs * desc->num_q_heads * sp.pmax;
    prm.ws_o = need ? static_cast<float *>(workspace) : nullptr;
    prm.ws_ml = need ? reinterpret_cast<float *>(static_cast<char *>(workspace) +
                                                 round_up(rows * desc->head_dim * 4, 256))
                     : nullptr;
    prm.S = desc->num_seqs;
    prm.Hq = desc->num_q_heads;
    prm.Hkv = desc->num_kv_heads;
    prm.NB = desc->num_blocks;
    prm.maxB = desc->max_blocks_per_seq;
    prm.part_blocks = sp.part_blocks;
    prm.pmax = sp.pmax;
    prm.scale_log2 = scale * 1.4426950408889634f;
    prm.bshift = block_shift(desc);
    prm.Lmax = (int32_t)lmax;
    const int g = desc->num_q_heads / desc->num_kv_heads;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (desc->dtype == PKV_F16)
        return desc->head_dim == 64 ? dispatch_group_tc<__half, 64, true>(g, prm, PKV_F16, s)
                                    : dispatch_group_tc<__half, 128, true>(g, prm, PKV_F16, s);
    return desc->head_dim == 64
               ? dispatch_group_tc<__nv_bfloat16, 64, true>(g, prm, PKV_BF16, s)
               : dispatch_group_tc<__nv_bfloat16, 128, true>(g, prm, PKV_BF16, s);
}

}  // extern "C"

// ---- FP8 (E4M3) KV cache --------------------------------------------------------------------
namespace {

#ifndef PKV_DECODE_FP8_STAGES
#define PKV_DECODE_FP8_STAGES 2
#endif
constexpr int kFp8Stages = PKV_DECODE_FP8_STAGES;  // blocks in flight per warp ring

// Warps per CTA: 4 for one query head per kv head (measured +5 % on the OPT-13B-shaped
// batch, whose mostly short partitions gain from more warps per unit), else 2 (4 cost 5 %
// on 512-token partitions at four heads per kv head).  PKV_DECODE_FP8_WARPS forces one.
template <int G>
constexpr int fp8_warps() {
#ifdef PKV_DECODE_FP8_WARPS
    return PKV_DECODE_FP8_WARPS;
#else
    return G == 1 ? 4 : 2;
#endif
}

pkv_status fp8_k_tensor_map(CUtensorMap *m, const void *pool, int64_t rows, const char *fn) {
    auto enc = tensor_map_encoder();
    if (!enc) return fail(PKV_ERR_CUDA, "%s: cuTensorMapEncodeTiled unavailable", fn);
    const cuuint64_t dims[2] = {128, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {128};
    const cuuint32_t box[2] = {128, (cuuint32_t)pkv::kBlock};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(pool), dims,
                     strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
        return fail(PKV_ERR_CUDA, "%s: cuTensorMapEncodeTiled failed (%d)", fn, (int)r);
    return PKV_OK;
}

template <typename T, int G, int BSH>
pkv_status launch_decode_fp8(const pkv::DecodeFp8Params &fp, cudaStream_t stream) {
    constexpr int kW = fp8_warps<G>();
    using Cfg = pkv::DecodeFp8Cfg<kW, kFp8Stages>;
    constexpr int kSmem = Cfg::template smem<G>();
    auto kern = pkv::paged_attn_decode_fp8_kernel<T, G, kW, kFp8Stages, BSH>;
    static std::atomic<bool> done[kMaxDevices];
    pkv_status st = ensure_smem(kern, kSmem, done, "paged_attn_decode_fp8");
    if (st) return st;
    CUtensorMap tmk;
    st = fp8_k_tensor_map(&tmk, fp.base.k_pool,
                          ((int64_t)fp.base.NB * fp.base.Hkv) << fp.base.bshift,
                          "paged_attn_decode_fp8");
    if (st) return st;
    const unsigned grid = (unsigned)((int64_t)fp.base.S * fp.base.Hkv * fp.base.pmax);
    kern<<<grid, kW * 32, kSmem, stream>>>(tmk, fp);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_check(e, "paged_attn_decode_fp8", "decode launch");
    return launch_reduce_if_split<T, 128>(fp.base, stream);
}

// The FP8 kernel takes the block size as a template parameter (16- or 32-token blocks).
template <typename T, int G>
pkv_status launch_decode_fp8_bs(const pkv::DecodeFp8Params &fp, cudaStream_t stream) {
    return fp.base.bshift == 5 ? launch_decode_fp8<T, G, 5>(fp, stream)
                               : launch_decode_fp8<T, G, 4>(fp, stream);
}

// Streaming multiprocessors of the current device (looked up once per device).
int device_sm_count() {
    static std::atomic<int> count[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
    int n = count[dev].load(std::memory_order_relaxed);
    if (n == 0 && cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess)
        count[dev].store(n, std::memory_order_relaxed);
    return n;
}

// The FP8 decode's partition when the caller leaves the choice to the library
// (partition_tokens 0).  Its per-unit work (the q conversion to f16, the warps' merge)
// weighs more against a unit's blocks than in the 16-bit kernel, so when the batch's
// (sequence, kv head) pairs alone give at least four CTAs per resident CTA slot it takes
// units of up to kFp8WidePartitionTokens (one per pair for contexts up to that), else the
// default 512.  Measured on the OPT-13B-shaped batch: +13 %.  Never more partitions than the
// default, so the default's workspace always suffices.
constexpr int32_t kFp8WidePartitionTokens = 2048;
// Resident warps per SM the choice counts with (fixed, so that the partition, and with it the
// rounding of the result, does not change when the kernel's occupancy is tuned).
constexpr int kFp8PartitionWarpsPerSm = 16;

Split fp8_split(const pkv_attn_desc *d, const Split &dflt) {
    if (d->partition_tokens != 0) return dflt;
    const int g = d->num_q_heads / d->num_kv_heads;
    const int warps = g == 1 ? fp8_warps<1>() : fp8_warps<2>();
    const int64_t slots = (int64_t)device_sm_count() * (kFp8PartitionWarpsPerSm / warps);
    const int64_t pairs = (int64_t)d->num_seqs * d->num_kv_heads;
    if (slots <= 0 || pairs < 4 * slots) return dflt;
    Split sp;
    sp.part_blocks = kFp8WidePartitionTokens / pkv::kBlock;
    sp.pmax = (sub_blocks_per_seq(d) + sp.part_blocks - 1) / sp.part_blocks;
    return sp.pmax < dflt.pmax ? sp : dflt;
}

template <typename T>
pkv_status dispatch_fp8(int g, const pkv::DecodeFp8Params &fp, cudaStream_t stream) {
    switch (g) {
    case 1: return launch_decode_fp8_bs<T, 1>(fp, stream);
    case 2: return launch_decode_fp8_bs<T, 2>(fp, stream);
    case 4: return launch_decode_fp8_bs<T, 4>(fp, stream);
    case 8: return launch_decode_fp8_bs<T, 8>(fp, stream);
    default: return fail(PKV_ERR_UNSUPPORTED, "paged_attn_decode_fp8: group %d", g);
    }
}

// Shared body of paged_attn_decode_fp8 and kv_write_fp8_and_decode (k_new / v_new /
// slot_mapping NULL: no fused write).
pkv_status decode_fp8_impl(const pkv_attn_desc *desc, const void *q, const void *k_new,
                           const void *v_new, const int64_t *slot_mapping, const void *k_pool,
                           const void *v_pool, const float *k_scale, const float *v_scale,
                           const int32_t *block_tables, const int32_t *context_lens,
                           float scale, void *out, void *workspace,
                           size_t workspace_bytes_given, void *stream, const char *fn) {
    Split sp;
    pkv_status st = check_attn_desc(desc, fn, &sp);
    if (st) return st;
    if (desc->dtype != PKV_F16 && desc->dtype != PKV_BF16)
        return fail(PKV_ERR_UNSUPPORTED, "%s: q/out must be f16 or bf16", fn);
    if (desc->head_dim != 128)
        return fail(PKV_ERR_UNSUPPORTED, "%s: only head_dim 128 is built", fn);
    if ((int64_t)desc->num_blocks * desc->num_kv_heads * desc->block_size >= ((int64_t)1 << 31))
        return fail(PKV_ERR_UNSUPPORTED, "%s: pool too large for 32-bit TMA rows", fn);
    if (desc->num_seqs == 0) return PKV_OK;
    if (!q || !k_pool || !v_pool || !k_scale || !v_scale || !block_tables || !context_lens ||
        !out)
        return fail(PKV_ERR_INVALID, "%s: NULL pointer", fn);
    if (!aligned(q, 16) || !aligned(k_pool, 16) || !aligned(v_pool, 16) || !aligned(out, 16) ||
        !aligned(k_scale, 4) || !aligned(v_scale, 4) || !aligned(block_tables, 4) ||
        !aligned(context_lens, 4))
        return fail(PKV_ERR_INVALID, "%s: misaligned pointer", fn);
    if (!std::isfinite(scale)) return fail(PKV_ERR_INVALID, "%s: scale is not finite", fn);
    const size_t need = workspace_bytes(desc, sp);
    if (need) {
        if (!workspace || workspace_bytes_given < need)
            return fail(PKV_ERR_INVALID, "%s: workspace needs %zu bytes", fn, need);
        if (!aligned(workspace, 256))
            return fail(PKV_ERR_INVALID, "%s: workspace must be 256-byte aligned", fn);
    }
    pkv::DecodeFp8Params fp;
    pkv::DecodeParams &prm = fp.base;
    prm.q = q;
    prm.k_pool = k_pool;
    prm.v_pool = v_pool;
    prm.k_new = k_new;
    prm.v_new = v_new;
    prm.slot_mapping = slot_mapping;
    prm.block_tables = block_tables;
    prm.context_lens = context_lens;
    prm.out = out;
    const Split run = fp8_split(desc, sp);
    const bool split = run.pmax > 1;
    const size_t rows = (size_t)desc->num_seqs * desc->num_q_heads * run.pmax;
    prm.ws_o = split ? static_cast<float *>(workspace) : nullptr;
    prm.ws_ml = split ? reinterpret_cast<float *>(static_cast<char *>(workspace) +
                                                  round_up(rows * desc->head_dim * 4, 256))
                      : nullptr;
    prm.S = desc->num_seqs;
    prm.Hq = desc->num_q_heads;
    prm.Hkv = desc->num_kv_heads;
    prm.NB = desc->num_blocks;
    prm.maxB = desc->max_blocks_per_seq;
    prm.part_blocks = run.part_blocks;
    prm.pmax = run.pmax;
    prm.scale_log2 = scale * 1.4426950408889634f;
    prm.bshift = block_shift(desc);
    fp.k_scale = k_scale;
    fp.v_scale = v_scale;
    const int g = desc->num_q_heads / desc->num_kv_heads;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (desc->dtype == PKV_F16) return dispatch_fp8<__half>(g, fp, s);
    return dispatch_fp8<__nv_bfloat16>(g, fp, s);
}

}  // namespace

extern "C" {

int32_t pkv_fp8_partition_tokens(const pkv_attn_desc *desc) {
    pkv::clear_error();
    Split sp;
    if (check_attn_desc(desc, "pkv_fp8_partition_tokens", &sp)) return 0;
    return fp8_split(desc, sp).part_blocks * pkv::kBlock;
}

pkv_status kv_write_fp8(const pkv_attn_desc *desc, const void *k_new, const void *v_new,
                        const int64_t *slot_mapping, int32_t num_tokens, const float *k_scale,
                        const float *v_scale, void *k_pool, void *v_pool, void *stream) {
    const char *fn = "kv_write_fp8";
    pkv_status st = check_pool_desc(desc, fn);
    if (st) return st;
    if (desc->dtype == PKV_FP8_E4M3)
        return fail(PKV_ERR_INVALID, "%s: desc->dtype is the type of the new values", fn);
    if (desc->head_dim != 128)
        return fail(PKV_ERR_UNSUPPORTED, "%s: only head_dim 128 is built", fn);
    if (num_tokens < 0) return fail(PKV_ERR_INVALID, "%s: num_tokens < 0", fn);
    if (num_tokens == 0) return PKV_OK;
    if (!k_new || !v_new || !slot_mapping || !k_scale || !v_scale || !k_pool || !v_pool)
        return fail(PKV_ERR_INVALID, "%s: NULL pointer", fn);
    if (!aligned(k_new, 16) || !aligned(v_new, 16) || !aligned(slot_mapping, 8) ||
        !aligned(k_scale, 4) || !aligned(v_scale, 4) || !aligned(k_pool, 16) ||
        !aligned(v_pool, 16))
        return fail(PKV_ERR_INVALID, "%s: misaligned pointer", fn);
    pkv::KvWriteFp8Params prm;
    prm.k_new = k_new;
    prm.v_new = v_new;
    prm.slot_mapping = slot_mapping;
    prm.k_scale = k_scale;
    prm.v_scale = v_scale;
    prm.k_pool = static_cast<uint8_t *>(k_pool);
    prm.v_pool = static_cast<uint8_t *>(v_pool);
    prm.T = num_tokens;
    prm.Hkv = desc->num_kv_heads;
    prm.NB = desc->num_blocks;
    prm.D = desc->head_dim;
    prm.bshift = block_shift(desc);
    dim3 grid;
    st = write_grid(num_tokens, (int64_t)prm.Hkv * (prm.D / 2), &grid, fn);
    if (st) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    constexpr int kT = pkv::kWriteThreads;
    switch (desc->dtype) {
    case PKV_F32: pkv::kv_write_fp8_kernel<float><<<grid, kT, 0, s>>>(prm); break;
    case PKV_F16: pkv::kv_write_fp8_kernel<__half><<<grid, kT, 0, s>>>(prm); break;
    default: pkv::kv_write_fp8_kernel<__nv_bfloat16><<<grid, kT, 0, s>>>(prm); break;
    }
    return cuda_check(cudaGetLastError(), fn, "launch");
}

pkv_status paged_attn_decode_fp8(const pkv_attn_desc *desc, const void *q, const void *k_pool,
                                 const void *v_pool, const float *k_scale,
                                 const float *v_scale, const int32_t *block_tables,
                                 const int32_t *context_lens, float scale, void *out,
                                 void *workspace, size_t workspace_bytes_given, void *stream) {
    return decode_fp8_impl(desc, q, nullptr, nullptr, nullptr, k_pool, v_pool, k_scale, v_scale,
                           block_tables, context_lens, scale, out, workspace,
                           workspace_bytes_given, stream, "paged_attn_decode_fp8");
}

pkv_status kv_write_fp8_and_decode(const pkv_attn_desc *desc, const void *q, const void *k_new,
                                   const void *v_new, const int64_t *slot_mapping,
                                   const float *k_scale, const float *v_scale, void *k_pool,
                                   void *v_pool, const int32_t *block_tables,
                                   const int32_t *context_lens, float scale, void *out,
                                   void *workspace, size_t workspace_bytes_given,
                                   void *stream) {
    const char *fn = "kv_write_fp8_and_decode";
    if (desc && desc->num_seqs > 0) {
        if (!k_new || !v_new || !slot_mapping)
            return fail(PKV_ERR_INVALID, "%s: NULL tensor pointer", fn);
        if (!aligned(k_new, 16) || !aligned(v_new, 16) || !aligned(slot_mapping, 8))
            return fail(PKV_ERR_INVALID, "%s: misaligned pointer", fn);
    }
    return decode_fp8_impl(desc, q, k_new, v_new, slot_mapping, k_pool, v_pool, k_scale, v_scale,
                           block_tables, context_lens, scale, out, workspace,
                           workspace_bytes_given, stream, fn);
}

}  // extern "C"

// ---- allocation-free decode ----------------------------------------------------------------
// Split-context scratch that ships inside the library: one copy per device that loads it.
// In host code the name below is only a host-side stand-in for the device array, never a
// device address; the device address comes from cudaGetSymbolAddress, once per device.
static __device__ __align__(256) unsigned char g_static_workspace[PKV_STATIC_WORKSPACE_BYTES];

namespace {

std::mutex g_static_ws_mutex;
void *g_static_ws_ptr[kMaxDevices] = {};

// Device address of the current device's copy of g_static_workspace (looked up on first use).
pkv_status static_workspace(void **ptr, const char *fn) {
    int dev = 0;
    pkv_status st = cuda_check(cudaGetDevice(&dev), fn, "cudaGetDevice");
    if (st) return st;
    if (dev < 0 || dev >= kMaxDevices) return fail(PKV_ERR_CUDA, "%s: device %d", fn, dev);
    std::lock_guard<std::mutex> lock(g_static_ws_mutex);
    if (!g_static_ws_ptr[dev]) {
        void *p = nullptr;
        st = cuda_check(cudaGetSymbolAddress(&p, g_static_workspace), fn,
                        "cudaGetSymbolAddress(static workspace)");
        if (st) return st;
        g_static_ws_ptr[dev] = p;
    }
    *ptr = g_static_ws_ptr[dev];
    return PKV_OK;
}

}  // namespace

extern "C" {

pkv_status paged_attn_decode_no_alloc(const pkv_attn_desc *desc, const void *q,
                                      const void *k_pool, const void *v_pool,
                                      const int32_t *block_tables,
                                      const int32_t *context_lens, float scale, void *out,
                                      void *stream) {
    const char *fn = "paged_attn_decode_no_alloc";
    Split sp;
    pkv_status st = check_attn_desc(desc, fn, &sp);
    if (st) return st;
    const size_t need = workspace_bytes(desc, sp);
    if (need > PKV_STATIC_WORKSPACE_BYTES)
        return fail(PKV_ERR_INVALID,
                    "%s: this batch needs %zu bytes of split scratch; the library's static "
                    "workspace holds %u (use paged_attn_decode with a workspace, fewer "
                    "sequences, or larger partition_tokens)",
                    fn, need, (unsigned)PKV_STATIC_WORKSPACE_BYTES);
    if (desc->num_seqs == 0) return PKV_OK;
    void *ws = nullptr;
    if (need) {
        st = static_workspace(&ws, fn);
        if (st) return st;
    }
    return paged_attn_decode(desc, q, k_pool, v_pool, block_tables, context_lens, scale, out,
                             ws, need ? (size_t)PKV_STATIC_WORKSPACE_BYTES : 0, stream);
}

}  // extern "C"

namespace {

// Device-side address of a caller's pinned host buffer; rejects memory the GPU cannot reach.
pkv_status mapped_host(const void *host, void **dev, const char *fn, const char *name) {
    cudaPointerAttributes a;
    cudaError_t e = cudaPointerGetAttributes(&a, host);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return fail(PKV_ERR_INVALID, "%s: %s is not a CUDA-registered host buffer", fn, name);
    }
    if (a.type != cudaMemoryTypeHost || !a.devicePointer)
        return fail(PKV_ERR_INVALID, "%s: %s must be pinned host memory mapped for the device",
                    fn, name);
    if (!aligned(a.devicePointer, 16))
        return fail(PKV_ERR_INVALID, "%s: %s must be 16-byte aligned", fn, name);
    *dev = a.devicePointer;
    return PKV_OK;
}

pkv_status launch_swap(const pkv_attn_desc *desc, const int32_t *pairs, int32_t n,
                       const void *src_k, const void *src_v, int32_t nb_src, void *dst_k,
                       void *dst_v, int32_t nb_dst, cudaStream_t stream, const char *fn) {
    if (n > INT_MAX / 2) return fail(PKV_ERR_INVALID, "%s: too many pairs", fn);
    pkv::KvSwapParams prm;
    prm.pairs = pairs;
    prm.src_k = static_cast<const uint4 *>(src_k);
    prm.src_v = static_cast<const uint4 *>(src_v);
    prm.dst_k = static_cast<uint4 *>(dst_k);
    prm.dst_v = static_cast<uint4 *>(dst_v);
    prm.P = n;
    prm.nb_src = nb_src;
    prm.nb_dst = nb_dst;
    prm.vpb = (int64_t)desc->num_kv_heads * desc->block_size * desc->head_dim *
              elem_size(desc->dtype) / 16;
    const int64_t slices = (prm.vpb + pkv::kCopyUnroll * 256 - 1) / (pkv::kCopyUnroll * 256);
    if (slices > 65535) return fail(PKV_ERR_UNSUPPORTED, "%s: block too large", fn);
    dim3 grid((unsigned)(2 * n), (unsigned)slices);
    pkv::kv_swap_kernel<<<grid, 256, 0, stream>>>(prm);
    return cuda_check(cudaGetLastError(), fn, "launch");
}

pkv_status check_swap_args(const pkv_attn_desc *desc, const int32_t *pairs, int32_t n,
                           const void *k_pool, const void *v_pool, const void *host_k,
                           const void *host_v, int32_t num_host_blocks, const char *fn) {
    pkv_status st = check_pool_desc(desc, fn);
    if (st) return st;
    if (n < 0 || num_host_blocks < 0) return fail(PKV_ERR_INVALID, "%s: negative size", fn);
    if (n > 0 && (!pairs || !k_pool || !v_pool || !host_k || !host_v))
        return fail(PKV_ERR_INVALID, "%s: NULL pointer", fn);
    if (n > 0 && (!aligned(k_pool, 16) || !aligned(v_pool, 16) || !aligned(pairs, 4)))
        return fail(PKV_ERR_INVALID, "%s: misaligned pointer", fn);
    return PKV_OK;
}

}  // namespace

extern "C" {

pkv_status kv_swap_out(const pkv_attn_desc *desc, const int32_t *pairs, int32_t num_pairs,
                       const void *k_pool, const void *v_pool, void *host_k, void *host_v,
                       int32_t num_host_blocks, void *stream) {
    const char *fn = "kv_swap_out";
    pkv_status st = check_swap_args(desc, pairs, num_pairs, k_pool, v_pool, host_k, host_v,
                                    num_host_blocks, fn);
    if (st || num_pairs == 0) return st;
    void *dk = nullptr, *dv = nullptr;
    if ((st = mapped_host(host_k, &dk, fn, "host_k")) || (st = mapped_host(host_v, &dv, fn,
                                                                              "host_v")))
        return st;
    return launch_swap(desc, pairs, num_pairs, k_pool, v_pool, desc->num_blocks, dk, dv,
                       num_host_blocks, static_cast<cudaStream_t>(stream), fn);
}

pkv_status kv_swap_in(const pkv_attn_desc *desc, const int32_t *pairs, int32_t num_pairs,
                      const void *host_k, const void *host_v, int32_t num_host_blocks,
                      void *k_pool, void *v_pool, void *stream) {
    const char *fn = "kv_swap_in";
    pkv_status st = check_swap_args(desc, pairs, num_pairs, k_pool, v_pool, host_k, host_v,
                                    num_host_blocks, fn);
    if (st || num_pairs == 0) return st;
    void *dk = nullptr, *dv = nullptr;
    if ((st = mapped_host(host_k, &dk, fn, "host_k")) || (st = mapped_host(host_v, &dv, fn,
                                                                              "host_v")))
        return st;
    return launch_swap(desc, pairs, num_pairs, dk, dv, num_host_blocks, k_pool, v_pool,
                       desc->num_blocks, static_cast<cudaStream_t>(stream), fn);
}

pkv_status pkv_device_faults(uint32_t *faults, int clear, void *stream) {
    const char *fn = "pkv_device_faults";
    if (!faults) return fail(PKV_ERR_INVALID, "%s: faults is NULL", fn);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    unsigned int *addr = nullptr;
    pkv_status st = cuda_check(cudaGetSymbolAddress((void **)&addr, pkv::g_faults), fn,
                               "cudaGetSymbolAddress");
    if (st) return st;
    unsigned int h = 0;
    st = cuda_check(cudaMemcpyAsync(&h, addr, sizeof(h), cudaMemcpyDeviceToHost, s), fn,
                    "read");
    if (st) return st;
    if (clear) {
        st = cuda_check(cudaMemsetAsync(addr, 0, sizeof(unsigned int), s), fn, "clear");
        if (st) return st;
    }
    st = cuda_check(cudaStreamSynchronize(s), fn, "synchronize");
    if (st) return st;
    *faults = h;
    return PKV_OK;
}

}  // extern "C"

// ---- read-bandwidth probe -------------------------------------------------------------------
extern "C" pkv_status pkv_read_probe(const void *buf, size_t bytes, int32_t chunk_bytes,
                                     int32_t ctas_per_sm, size_t *bytes_read, void *stream) {
    const char *fn = "pkv_read_probe";
    if (!buf || (reinterpret_cast<uintptr_t>(buf) & 15u))
        return fail(PKV_ERR_INVALID, "%s: buf null or not 16-byte aligned", fn);
    if (chunk_bytes != 2048 && chunk_bytes != 4096 && chunk_bytes != 8192 &&
        chunk_bytes != 16384)
        return fail(PKV_ERR_INVALID, "%s: chunk_bytes %d (2048, 4096, 8192 or 16384)", fn,
                    chunk_bytes);
    const uint64_t chunks = bytes / (uint64_t)chunk_bytes;
    if (chunks < 1 || chunks > (1ull << 31))
        return fail(PKV_ERR_INVALID, "%s: %llu chunks (1 .. 2^31)", fn,
                    (unsigned long long)chunks);
    uint64_t n = 1;
    while (n * 2 <= chunks) n *= 2;
    const int smem = pkv::kProbeWarps * pkv::kProbeStages * chunk_bytes +
                     pkv::kProbeWarps * pkv::kProbeStages * 8;
    // the shared-memory limit is set once per device, for the largest chunk
    const int smem_max = pkv::kProbeWarps * pkv::kProbeStages * 16384 +
                         pkv::kProbeWarps * pkv::kProbeStages * 8;
    static std::atomic<bool> done[kMaxDevices];
    pkv_status st = ensure_smem(pkv::read_probe_kernel, smem_max, done, fn);
    if (st) return st;
    int per_sm = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(
        &per_sm, pkv::read_probe_kernel, pkv::kProbeWarps * 32, smem);
    if (e != cudaSuccess) return cuda_check(e, fn, "occupancy");
    const int sms = device_sm_count();
    if (per_sm < 1 || sms < 1) return fail(PKV_ERR_CUDA, "%s: no resident CTA fits", fn);
    if (ctas_per_sm < 0) return fail(PKV_ERR_INVALID, "%s: ctas_per_sm %d", fn, ctas_per_sm);
    if (ctas_per_sm > 0) per_sm = ctas_per_sm;   // more than fit simply run in turns
    const uint32_t grid = (uint32_t)sms * (uint32_t)per_sm;
    pkv::read_probe_kernel<<<grid, pkv::kProbeWarps * 32, smem,
                             static_cast<cudaStream_t>(stream)>>>(
        static_cast<const char *>(buf), (uint32_t)n, (uint32_t)chunk_bytes);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_check(e, fn, "launch");
    if (bytes_read) *bytes_read = (size_t)(n * (uint64_t)chunk_bytes);
    return PKV_OK;
}
