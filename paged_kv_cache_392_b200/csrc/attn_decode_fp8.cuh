// FP8 (E4M3) paged KV cache: quantising write and tensor-core decode (sm_100a).
//
// "Memory Optimization in LLM Serving with PagedAttention", section "Broader Context: vLLM,
// TGI, and TensorRT-LLM": paged KV caches are also kept in INT8/FP8 to cut memory.  The page
// fixes no format; this library's reading:
//   * each KV head has one fp32 scale for K and one for V; element x is stored as the E4M3
//     code of x / scale (fp32 division, round to nearest even, saturating to +-448) and
//     means code * scale;
//   * K blocks: [block][kv head][B tokens][D] bytes (as the 16-bit pools), B = 16 or 32;
//   * V blocks: [block][kv head][B/16][D][16 slots] bytes -- each 16-token half of a block
//     transposed, and slot p of a row holds token 2*(p>>2) + (p&1) + 8*((p>>1)&1) of the
//     half (v_slot_of_token below is the inverse), so that the 4 bytes an ldmatrix lane
//     reads from a row are the token pairs the P.V tile wants.
// Decode: q.K^T and P.V run on m16n8k16 f16 tensor-core tiles.  Every E4M3 value is an f16
// value, so the K and V codes are widened exactly, four codes (two f16x2 registers) per
// conversion pair; q enters as f16 (an f16 q as is, a bf16 q scaled by a power of two, which
// rounds it to f16 exactly).  Accumulation is fp32; the K scale (and the q scale) is folded
// into the softmax scale and the V scale into the output.  Only D = 128 is built.
#pragma once
#include <cuda.h>
#include <cuda_fp8.h>

#include <type_traits>

#include "attn_decode_tc.cuh"
#include "kv_ops.cuh"

namespace pkv {

// Slot p of a transposed V row holds token t = 2*(p>>2) + (p&1) + 8*((p>>1)&1); its inverse:
__host__ __device__ __forceinline__ int v_slot_of_token(int t) {
    return 4 * ((t & 7) >> 1) + 2 * (t >> 3) + (t & 1);
}

// Tuning switch of the FP8 decode (the results are the same bits either way): 1 computes
// the softmax weights before the rescale vote resolves (measured +0.4 to +1.4 %).
#ifndef PKV_FP8_SPEC_EXP
#define PKV_FP8_SPEC_EXP 1
#endif

// Four E4M3 codes (bytes 0..3 of w) to two f16x2 registers, exactly: lo = codes 0, 1 and
// hi = codes 2, 3, each pair with its lower-addressed code in the low half.  The conversion
// reads the 16-bit halves of w directly (one instruction per output register).
__device__ __forceinline__ void e4m3x4_to_f16x2x2(uint32_t w, uint32_t &lo, uint32_t &hi) {
    asm("{\n\t.reg .b16 l, h;\n\t"
        "mov.b32 {l, h}, %2;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, l;\n\t"
        "cvt.rn.f16x2.e4m3x2 %1, h;\n\t}"
        : "=r"(lo), "=r"(hi)
        : "r"(w));
}

// Two floats to an f16x2 register (round to nearest even).
__device__ __forceinline__ uint32_t f32x2_to_f16x2(float lo, float hi) {
    return pack2<false>(lo, hi);
}

struct DecodeFp8Params {
    DecodeParams base;        // q/out/workspace/shape (k_pool/v_pool: the E4M3 pools)
    const float *k_scale;     // [H_kv]
    const float *v_scale;     // [H_kv]
};

template <typename T>
__device__ __forceinline__ float load_elem(const void *base, int64_t i) {
    if constexpr (std::is_same<T, float>::value)
        return static_cast<const float *>(base)[i];
    else if constexpr (std::is_same<T, __half>::value)
        return __half2float(static_cast<const __half *>(base)[i]);
    else
        return __bfloat162float(static_cast<const __nv_bfloat16 *>(base)[i]);
}

// Whether an FP8 scale can encode: finite and above zero (NaN fails both tests).
__device__ __forceinline__ bool scale_ok(float x) { return x > 0.f && x < INFINITY; }

// E4M3 codes of src[i] / scale and src[i+1] / scale (fp32 division, round to nearest even,
// saturating to +-448), element i in the low byte: the cache format's quantisation.
template <typename T>
__device__ __forceinline__ __nv_fp8x2_storage_t quantize2(const void *src, int64_t i,
                                                         float scale) {
    const float2 x = make_float2(load_elem<T>(src, i) / scale, load_elem<T>(src, i + 1) / scale);
    return __nv_cvt_float2_to_fp8x2(x, __NV_SATFINITE, __NV_E4M3);
}

// Fused kv_write_fp8 of sequence s's newest token for kv head hk, by the one warp that will
// copy the block holding position L-1: quantise the K row and the V column into their slot,
// then fence the generic-proxy stores against the warp's own TMA / bulk copies of the block.
// A slot of -1 is skipped; any slot other than position L-1's sets fault bit 4 (bad slot)
// and is not written, and neither is anything when the head's K or V scale is not finite
// and > 0 (fault bit 0x40).
template <typename T, int BSH>
__device__ __forceinline__ void write_newest_token_fp8(const DecodeFp8Params &fp, int s, int hk,
                                                       int L, int lane) {
    constexpr int D = 128;
    const DecodeParams &p = fp.base;
    const int64_t slot = p.slot_mapping[s];
    if (slot != -1) {
        const int32_t blk = p.block_tables[(size_t)s * p.maxB + ((L - 1) >> BSH)];
        const int off = (L - 1) & ((1 << BSH) - 1);
        const float ksc = fp.k_scale[hk], vsc = fp.v_scale[hk];
        if (!scale_ok(ksc) || !scale_ok(vsc)) {
            if (lane == 0) atomicOr(&g_faults, kFaultBadScale);
        } else if ((unsigned)blk < (unsigned)p.NB && slot == ((int64_t)blk << BSH) + off) {
            const int64_t src = ((int64_t)s * p.Hkv + hk) * D;
            const int64_t hb = (int64_t)blk * p.Hkv + hk;
            // the 16-token half of the block that holds the token, and its V^T slot
            const int64_t vh = (hb << (BSH - 4)) + (off >> 4);
            const int vs = v_slot_of_token(off & 15);
            // the pools are written only here; the decode itself reads them
            uint8_t *kp = static_cast<uint8_t *>(const_cast<void *>(p.k_pool));
            uint8_t *vp = static_cast<uint8_t *>(const_cast<void *>(p.v_pool));
            for (int d = 2 * lane; d < D; d += 64) {
                const __nv_fp8x2_storage_t kc = quantize2<T>(p.k_new, src + d, ksc);
                const __nv_fp8x2_storage_t vc = quantize2<T>(p.v_new, src + d, vsc);
                *reinterpret_cast<__nv_fp8x2_storage_t *>(kp + ((hb << BSH) + off) * D +
                                                          d) = kc;
                vp[(vh * D + d) * kBlock + vs] = static_cast<uint8_t>(vc & 0xffu);
                vp[(vh * D + d + 1) * kBlock + vs] = static_cast<uint8_t>(vc >> 8);
            }
            fence_proxy_async_global();
        } else if (lane == 0) {
            atomicOr(&g_faults,
                     (unsigned)blk < (unsigned)p.NB ? kFaultBadSlot : kFaultBadBlock);
        }
    }
    __syncwarp();
}

template <int W, int NSW>
struct DecodeFp8Cfg {
    static constexpr int D = 128;
    static constexpr int CHUNK = kBlock * D;      // bytes of one (block, head) of K or of V
    static constexpr int STAGE = 2 * CHUNK;       // K (swizzled box) then V (transposed)
    static constexpr int RING = W * NSW * STAGE;
    static constexpr int BARS = W * NSW * 8;
    static constexpr int KSTEPS = D / 16;
    // the warps' merge states [W][G][D] + [W][G][2] floats reuse the ring once every warp
    // is done with it
    template <int G>
    static constexpr int smem() {
        static_assert(W * G * (D + 2) * 4 <= RING, "merge states must fit in the ring");
        return 1024 + RING + BARS;
    }
};

// Resident warps per SM the register cap is sized for.  With 18, the 2-warp CTAs compile to
// 96 registers (10 CTAs per SM) and the 4-warp CTAs (one query head per kv head) to 124 (4
// per SM); 16 and 20 measured 1-4 % slower on the grouped-head batches, 24 spills.
#ifndef PKV_FP8_WARPS_PER_SM
#define PKV_FP8_WARPS_PER_SM 18
#endif
constexpr int kFp8WarpsPerSm = PKV_FP8_WARPS_PER_SM;

// T: the q / out type (__half or __nv_bfloat16); the pools are E4M3 bytes.  G query heads
// per kv head, W warps per CTA, NSW ring stages per warp, BSH log2 of the tokens per physical
// block (4 or 5: a compile-time constant here, so that the block addressing of the 16-token
// blocks costs nothing; it must equal DecodeParams::bshift).
template <typename T, int G, int W, int NSW, int BSH>
__global__ void __launch_bounds__(W * 32, kFp8WarpsPerSm / W)
paged_attn_decode_fp8_kernel(const __grid_constant__ CUtensorMap tmk,
                             const DecodeFp8Params fp) {
    using C = DecodeFp8Cfg<W, NSW>;
    constexpr int D = C::D, CHUNK = C::CHUNK, KSTEPS = C::KSTEPS;
    constexpr unsigned FULL = 0xffffffffu;
    const DecodeParams &p = fp.base;

    extern __shared__ unsigned char smem_raw[];
    unsigned char *smem = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

    pdl_launch_dependents();

    const int bid = blockIdx.x;
    const int part = bid % p.pmax;
    const int rest = bid / p.pmax;
    const int hk = rest % p.Hkv;
    const int s = rest / p.Hkv;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int g = lane >> 2;
    const int tq = lane & 3;
    const int j0 = part * p.part_blocks;
    const int32_t *btab = p.block_tables + (size_t)s * p.maxB;
    const int j1 = j0 + warp;  // this warp's first sub-block

    // Loads that need no context length start with it, so that a unit's start costs one
    // round trip less: this lane's query values (four 16-bit values a load) and the warp's
    // first 32 table entries (entries past the sequence's end lie inside its table row and
    // are never used).
    constexpr int K32 = D / 32;
    const bool hv = g < G;
    uint2 qraw[K32][2];
    {
        const T *qrow =
            static_cast<const T *>(p.q) + ((size_t)s * p.Hq + hk * G + (hv ? g : 0)) * D;
#pragma unroll
        for (int j = 0; j < K32; ++j)
#pragma unroll
            for (int b = 0; b < 2; ++b)
                qraw[j][b] = hv ? *reinterpret_cast<const uint2 *>(qrow + 32 * j + 16 * b + 4 * tq)
                                : make_uint2(0u, 0u);
    }
    int32_t tab;
    {
        const int e = sub_to_entry(j1 + W * lane, BSH);
        tab = e < p.maxB ? btab[e] : 0;
    }

    const int L = p.context_lens[s];
    if (L < 1 || L > (p.maxB << BSH)) {
        if (part == 0 && hk == 0 && threadIdx.x == 0) atomicOr(&g_faults, kFaultBadLen);
        return;
    }
    const int nblk = (L + kBlock - 1) / kBlock;
    const int nparts = (nblk + p.part_blocks - 1) / p.part_blocks;
    if (part >= nparts) return;
    const int nb = min(nblk, j0 + p.part_blocks) - j0;
    const int nbw = nb > warp ? (nb - warp + W - 1) / W : 0;

    unsigned char *ring = smem + warp * NSW * C::STAGE;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::RING) + warp * NSW;
    float *mo = reinterpret_cast<float *>(smem);  // over the ring, after the block loop
    float *mml = mo + W * G * D;

    if (lane == 0) {
#pragma unroll
        for (int i = 0; i < NSW; ++i) mbar_init(&bars[i], 1);
        fence_mbar_init();
        if (warp == 0) prefetch_tmap(&tmk);
    }
    __syncwarp();
    if (p.slot_mapping != nullptr && part == nparts - 1 && warp == (nb - 1) % W)
        write_newest_token_fp8<T, BSH>(fp, s, hk, L, lane);

    const char *vbase = static_cast<const char *>(p.v_pool);
    const uint64_t policy = l2_evict_first_policy();
    int tab_chunk = 0;

    auto issue = [&](int i) {
        if ((i >> 5) != tab_chunk) {
            tab_chunk = i >> 5;
            const int li = (tab_chunk << 5) + lane;
            tab = li < nbw ? btab[sub_to_entry(j1 + W * li, BSH)] : 0;
        }
        const int32_t phys = __shfl_sync(FULL, tab, i & 31);
        if (lane == 0 && !withheld_for_test(i, warp)) {
            uint64_t *bar = &bars[i % NSW];
            unsigned char *dst = ring + (i % NSW) * C::STAGE;
            if ((unsigned)phys < (unsigned)p.NB) {
                const int jb = j1 + W * i;
                const int32_t row = ((phys * p.Hkv + hk) << BSH) + sub_row(jb, BSH);
                // V^T of the sub-block: the 16-token half (jb's position in the block) of
                // the block's [B/16][D][16] bytes
                const size_t vhalf = ((size_t)(phys * p.Hkv + hk) << (BSH - 4)) +
                                     (size_t)(sub_row(jb, BSH) / kBlock);
                fence_proxy_async_smem();
                mbar_arrive_expect_tx(bar, 2 * CHUNK);
                tma_load_2d(dst, &tmk, 0, row, bar, policy);
                bulk_g2s(dst + CHUNK, vbase + vhalf * CHUNK, CHUNK, bar, policy);
            } else {
                atomicOr(&g_faults, kFaultBadBlock);
                mbar_arrive(bar);
            }
        }
    };

    const int npro = nbw < NSW ? nbw : NSW;
    for (int i = 0; i < npro; ++i) issue(i);
    int issued = npro;

    // Q^T as the B operand of S^T = K Q^T on f16 tiles (m16n8k16).  A K register from the
    // swizzled stage holds 4 consecutive dims of one token (the A fragment of an E4M3
    // m16n8k32 tile: lane (g, tq) reads dims 32j+4tq.. and 32j+16+4tq.. of tokens g and
    // g+8); widened, its dims d, d+1 and d+2, d+3 fill the f16 tile's k slots (2tq, 2tq+1)
    // and (2tq+8, 2tq+9).  The B fragment holds q at the same dims, so each tile sums q.k
    // over the 16 dims it covers: lane (g, tq) holds head g, dims 32j+16b+4tq..+3 as
    // qh[j][b][0] (the first two) and qh[j][b][1].  A bf16 q row is scaled by a power of two
    // qf (its largest |q| lands in [2^14, 2^15)), so that f16 holds every value exactly
    // except those 2^-28 below the row's largest; an f16 q is used as is.
    uint32_t qh[K32][2][2];
    float qf_mine = 1.f;
    {
        float qv[K32][2][4];
        float amax = 0.f;
#pragma unroll
        for (int j = 0; j < K32; ++j)
#pragma unroll
            for (int b = 0; b < 2; ++b) {
                const uint32_t w[2] = {qraw[j][b].x, qraw[j][b].y};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const uint16_t bits = static_cast<uint16_t>(w[e >> 1] >> (16 * (e & 1)));
                    float v;
                    if constexpr (std::is_same<T, __half>::value)
                        v = __half2float(__ushort_as_half(bits));
                    else
                        v = __bfloat162float(__ushort_as_bfloat16(bits));
                    qv[j][b][e] = v;
                    amax = fmaxf(amax, fabsf(v));
                }
            }
        if constexpr (!std::is_same<T, __half>::value) {
            amax = fmaxf(amax, __shfl_xor_sync(FULL, amax, 1));
            amax = fmaxf(amax, __shfl_xor_sync(FULL, amax, 2));
            if (amax > 0.f && amax < INFINITY) {
                int ex;
                frexpf(amax, &ex);                  // amax < 2^ex
                qf_mine = ldexpf(1.f, 15 - ex);     // amax * qf in [2^14, 2^15)
            }
        }
#pragma unroll
        for (int j = 0; j < K32; ++j)
#pragma unroll
            for (int b = 0; b < 2; ++b) {
                qh[j][b][0] = f32x2_to_f16x2(qv[j][b][0] * qf_mine, qv[j][b][1] * qf_mine);
                qh[j][b][1] = f32x2_to_f16x2(qv[j][b][2] * qf_mine, qv[j][b][3] * qf_mine);
            }
    }

    float o[KSTEPS][4];
#pragma unroll
    for (int i = 0; i < KSTEPS; ++i)
#pragma unroll
        for (int e = 0; e < 4; ++e) o[i][e] = 0.f;
    float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
    // score scales of this lane's heads 2tq, 2tq+1: softmax scale * K scale / q prescale
    if (threadIdx.x == 0 && (!scale_ok(fp.k_scale[hk]) || !scale_ok(fp.v_scale[hk])))
        atomicOr(&g_faults, kFaultBadScale);  // the output of this unit is then unspecified
    const float slk = p.scale_log2 * fp.k_scale[hk];
    const float sl0 = slk / __shfl_sync(FULL, qf_mine, (2 * tq) * 4);
    const float sl1 = slk / __shfl_sync(FULL, qf_mine, (2 * tq + 1) * 4);

    // ldmatrix roles.  K rows (tokens) in natural order; matrix mi of a k-step pair covers
    // tokens 8*(mi&1).. and 16-byte chunk 2j+(mi>>1).  V^T rows are head dims, two m-tiles
    // (32 rows) per x4.
    const int k_tok = (lane & 7) + 8 * ((lane >> 3) & 1);
    const int k_c = lane >> 4;
    const int v_row = lane;  // row within the 32-row group

    bool dead = false;
    int i = 0;
    for (; i < nbw; ++i) {
        const int st = i % NSW;
        if (!mbar_wait_bounded(&bars[st], (uint32_t)(i / NSW) & 1u, kWaitTimeoutNs)) {
            if (lane == 0) atomicOr(&g_faults, kFaultTimeout);
            dead = true;
            break;
        }
        unsigned char *Ks = ring + st * C::STAGE;
        unsigned char *Vs = Ks + CHUNK;
        const int jb = j0 + warp + W * i;
        const int nvalid = min(kBlock, L - jb * kBlock);
        if (nvalid < kBlock) {
            // zero the V^T slots of tokens past the context (their codes may be NaN)
            uint32_t keep[4] = {0u, 0u, 0u, 0u};
#pragma unroll
            for (int t = 0; t < kBlock; ++t)
                if (t < nvalid) {
                    const int sp = v_slot_of_token(t);
                    keep[sp >> 2] |= 0xffu << (8 * (sp & 3));
                }
            for (int r = lane; r < D; r += 32) {
                uint4 *row = reinterpret_cast<uint4 *>(Vs + r * 16);
                uint4 v = *row;
                v.x &= keep[0];
                v.y &= keep[1];
                v.z &= keep[2];
                v.w &= keep[3];
                *row = v;
            }
            fence_proxy_async_smem();
            __syncwarp();
        }

        // ---- the whole stage into registers: the K codes as the A fragments of S^T (row
        // g / g+8, k 4tq..4tq+3 and 16+4tq..16+4tq+3 of each 32-dim step) and the V^T rows
        // (r[0]: dims 32t2+0..7, r[1]: +8..15 of m-tile 2t2; r[2], r[3]: m-tile 2t2+1)
        uint32_t ka[K32][4], vr[KSTEPS / 2][4];
        const uint32_t kb = smem_u32(Ks);
#pragma unroll
        for (int j = 0; j < K32; ++j) {
            const int c = 2 * j + k_c;  // 16-byte chunk of the 128-byte row
            ldmatrix_x4(ka[j], kb + k_tok * 128 + ((c ^ (k_tok & 7)) << 4));
        }
        const uint32_t vb = smem_u32(Vs);
#pragma unroll
        for (int t2 = 0; t2 < KSTEPS / 2; ++t2) ldmatrix_x4(vr[t2], vb + (32 * t2 + v_row) * 16);

        // ---- S^T = K Q^T on f16 tiles: per 32-dim step, the tile of dims 32j+4tq.. and the
        // tile of dims 32j+16+4tq..
        float sacc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int j = 0; j < K32; ++j)
#pragma unroll
            for (int b = 0; b < 2; ++b) {
                uint32_t a[4];
                e4m3x4_to_f16x2x2(ka[j][2 * b], a[0], a[2]);      // token g
                e4m3x4_to_f16x2x2(ka[j][2 * b + 1], a[1], a[3]);  // token g + 8
                mma_16816<false>(sacc, a, qh[j][b][0], qh[j][b][1]);
            }

        // ---- online softmax (lane: tokens g, g+8 of heads 2tq, 2tq+1) --------------------
        float x0 = sacc[0] * sl0, x1 = sacc[1] * sl1, x2 = sacc[2] * sl0, x3 = sacc[3] * sl1;
        if (nvalid < kBlock) {  // the sequence's last block: no weight past its end
            x0 = g < nvalid ? x0 : -INFINITY;
            x1 = g < nvalid ? x1 : -INFINITY;
            x2 = g + 8 < nvalid ? x2 : -INFINITY;
            x3 = g + 8 < nvalid ? x3 : -INFINITY;
        }
        // Lazy rescale: a head's reference max moves only when a block's max passes it by
        // more than kLazyRescale (base 2), so P stays <= 2^kLazyRescale (f16 holds it); O / l
        // does not depend on the reference.  One vote tells whether any score passes its
        // reference by that much; only then (a warp's first block, and rarely after) does
        // the warp reduce the block's max and rescale O and its partial sums.
#if PKV_FP8_SPEC_EXP
        // The weights against the current references start before the vote resolves; the
        // rare block that moves a reference computes them again.
        float p0 = ex2_ftz(x0 - m_run[0]), p1 = ex2_ftz(x1 - m_run[1]);
        float p2 = ex2_ftz(x2 - m_run[0]), p3 = ex2_ftz(x3 - m_run[1]);
#endif
        if (__any_sync(FULL, fmaxf(x0, x2) > m_run[0] + kLazyRescale ||
                                 fmaxf(x1, x3) > m_run[1] + kLazyRescale)) {
            float bm0 = fmaxf(x0, x2), bm1 = fmaxf(x1, x3);
#pragma unroll
            for (int m = 4; m < 32; m <<= 1) {
                bm0 = fmaxf(bm0, __shfl_xor_sync(FULL, bm0, m));
                bm1 = fmaxf(bm1, __shfl_xor_sync(FULL, bm1, m));
            }
            const float mn0 = bm0 > m_run[0] + kLazyRescale ? bm0 : m_run[0];
            const float mn1 = bm1 > m_run[1] + kLazyRescale ? bm1 : m_run[1];
            const float a0 = mn0 == m_run[0] ? 1.f : ex2_ftz(m_run[0] - mn0);
            const float a1 = mn1 == m_run[1] ? 1.f : ex2_ftz(m_run[1] - mn1);
            l_run[0] *= a0;
            l_run[1] *= a1;
#pragma unroll
            for (int t = 0; t < KSTEPS; ++t) {
                o[t][0] *= a0;
                o[t][1] *= a1;
                o[t][2] *= a0;
                o[t][3] *= a1;
            }
            m_run[0] = mn0;
            m_run[1] = mn1;
#if PKV_FP8_SPEC_EXP
            p0 = ex2_ftz(x0 - m_run[0]);
            p1 = ex2_ftz(x1 - m_run[1]);
            p2 = ex2_ftz(x2 - m_run[0]);
            p3 = ex2_ftz(x3 - m_run[1]);
#endif
        }
#if !PKV_FP8_SPEC_EXP
        const float p0 = ex2_ftz(x0 - m_run[0]), p1 = ex2_ftz(x1 - m_run[1]);
        const float p2 = ex2_ftz(x2 - m_run[0]), p3 = ex2_ftz(x3 - m_run[1]);
#endif
        // per-lane partial sums; the 8 token-row lanes of a head add theirs after the loop
        l_run[0] += p0 + p2;
        l_run[1] += p1 + p3;

        // P^T fragments: b0 holds tokens 2tq, 2tq+1 and b1 tokens 8+2tq, 9+2tq of head g,
        // which are the slots 4tq..4tq+3 a lane reads from a V^T row.
        const uint32_t b0 = movmatrix_trans(f32x2_to_f16x2(p0, p1));
        const uint32_t b1 = movmatrix_trans(f32x2_to_f16x2(p2, p3));

        // ---- O^T += V^T P^T -----------------------------------------------------------------
#pragma unroll
        for (int t2 = 0; t2 < KSTEPS / 2; ++t2) {
            const uint32_t(&r)[4] = vr[t2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                uint32_t a[4];
                e4m3x4_to_f16x2x2(r[2 * h], a[0], a[2]);
                e4m3x4_to_f16x2x2(r[2 * h + 1], a[1], a[3]);
                mma_16816<false>(o[2 * t2 + h], a, b0, b1);
            }
        }
        __syncwarp();
        if (issued < nbw) {
            issue(issued);
            ++issued;
        }
    }
    if (dead) {
        for (int b = i; b < issued; ++b)
            (void)mbar_wait_bounded(&bars[b % NSW], (uint32_t)(b / NSW) & 1u, kWaitTimeoutNs);
        m_run[0] = m_run[1] = -INFINITY;
        l_run[0] = l_run[1] = 0.f;
#pragma unroll
        for (int t = 0; t < KSTEPS; ++t)
#pragma unroll
            for (int e = 0; e < 4; ++e) o[t][e] = 0.f;
    }

#pragma unroll
    for (int m = 4; m < 32; m <<= 1) {
        l_run[0] += __shfl_xor_sync(FULL, l_run[0], m);
        l_run[1] += __shfl_xor_sync(FULL, l_run[1], m);
    }

    __syncthreads();  // every warp is done with its ring: the merge states go over it
    const float vsc = fp.v_scale[hk];
    const int h0 = 2 * tq, h1 = 2 * tq + 1;
    if (h0 < G) {
        float *dst = mo + (warp * G + h0) * D;
#pragma unroll
        for (int t = 0; t < KSTEPS; ++t) {
            dst[16 * t + g] = o[t][0] * vsc;
            dst[16 * t + g + 8] = o[t][2] * vsc;
        }
        if (g == 0) {
            mml[(warp * G + h0) * 2] = m_run[0];
            mml[(warp * G + h0) * 2 + 1] = l_run[0];
        }
    }
    if (h1 < G) {
        float *dst = mo + (warp * G + h1) * D;
#pragma unroll
        for (int t = 0; t < KSTEPS; ++t) {
            dst[16 * t + g] = o[t][1] * vsc;
            dst[16 * t + g + 8] = o[t][3] * vsc;
        }
        if (g == 0) {
            mml[(warp * G + h1) * 2] = m_run[1];
            mml[(warp * G + h1) * 2 + 1] = l_run[1];
        }
    }
    __syncthreads();
    merge_and_store<T, D, G, W>(p, mo, mml, s, hk, part, nparts);
}

// ---- quantising write ----------------------------------------------------------------------
struct KvWriteFp8Params {
    const void *k_new;  // [T][H_kv][D] of the new-value type
    const void *v_new;
    const int64_t *slot_mapping;
    const float *k_scale;
    const float *v_scale;
    uint8_t *k_pool;    // [NB][H_kv][B][D]
    uint8_t *v_pool;    // [NB][H_kv][B/16][D][16] (slot order v_slot_of_token)
    int32_t T, Hkv, NB, D;
    int32_t bshift;     // log2 B (4 or 5)
};


// grid.x = tile of kTileTokens tokens, grid.y = slice of the tile's (token, head, pair of
// dims) items, one thread per item: codes of x / scale, RNE, saturating.  Slots shared by
// two tokens of the call are skipped (PKV_FAULT_DUPLICATE), as in kv_write; a head whose K
// or V scale is not finite and > 0 is not written (PKV_FAULT_BAD_SCALE).
template <typename T>
__global__ void __launch_bounds__(kWriteThreads) kv_write_fp8_kernel(const KvWriteFp8Params p) {
    __shared__ TileSlots ts;
    const int64_t t0 = (int64_t)blockIdx.x * kTileTokens;
    tile_duplicate_slots(p.slot_mapping, p.T, t0, ts);
    const int ntok = (int)(p.T - t0 < kTileTokens ? p.T - t0 : kTileTokens);
    const int per_tok = p.Hkv * (p.D / 2);
    const int items = ntok * per_tok;
    const int per_cta = (items + gridDim.y - 1) / gridDim.y;
    const int end = min(items, (int)(blockIdx.y + 1) * per_cta);
    for (int i = blockIdx.y * per_cta + threadIdx.x; i < end; i += kWriteThreads) {
        const int tl = i / per_tok, hd = i % per_tok;
        const int h = hd / (p.D / 2), d = 2 * (hd % (p.D / 2));
        const int64_t slot = ts.slot[tl];
        if (slot == -1) continue;
        if (slot < 0 || slot >= ((int64_t)p.NB << p.bshift)) {
            if (hd == 0) atomicOr(&g_faults, kFaultBadSlot);
            continue;
        }
        if ((ts.dup_mask >> tl) & 1u) {
            if (hd == 0) atomicOr(&g_faults, kFaultDuplicate);
            continue;
        }
        const float ksc = p.k_scale[h], vsc = p.v_scale[h];
        if (!scale_ok(ksc) || !scale_ok(vsc)) {
            if (d == 0) atomicOr(&g_faults, kFaultBadScale);
            continue;
        }
        const int64_t blk = slot >> p.bshift;
        const int off = (int)(slot & ((1 << p.bshift) - 1));
        const int64_t src = ((t0 + tl) * p.Hkv + h) * p.D + d;
        const __nv_fp8x2_storage_t kc = quantize2<T>(p.k_new, src, ksc);
        const __nv_fp8x2_storage_t vc = quantize2<T>(p.v_new, src, vsc);
        const int64_t hb = blk * p.Hkv + h;
        *reinterpret_cast<__nv_fp8x2_storage_t *>(p.k_pool + ((hb << p.bshift) + off) * p.D +
                                                  d) = kc;
        const int64_t vh = (hb << (p.bshift - 4)) + (off >> 4);  // the token's 16-token half
        const int sp = v_slot_of_token(off & 15);
        p.v_pool[(vh * p.D + d) * 16 + sp] = static_cast<uint8_t>(vc & 0xffu);
        p.v_pool[(vh * p.D + d + 1) * 16 + sp] = static_cast<uint8_t>(vc >> 8);
    }
}

}  // namespace pkv
