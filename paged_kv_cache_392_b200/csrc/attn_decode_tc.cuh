// Paged decode attention on the tensor cores (16-bit K/V, sm_100a).
//
// Same work decomposition, outputs and split/merge contract as paged_attn_decode_kernel
// (attn_decode.cuh); what changes is how one warp turns a staged 16-token block into scores
// and output.  The CUDA-core kernel spends ~1100 warp instructions per block when four query
// heads share a kv head (dot products, shuffle reductions, conversions), which leaves it
// issue-bound well below HBM bandwidth.  Here both contractions of the block are
// m16n8k16 tensor-core tiles, ~16 MMAs and ~16 ldmatrix per block:
//
//   S^T[16 tokens x 8] = K[16 x D] . Q^T[D x 8]      (the group's <= 8 query heads are the
//                                                    n columns; Q^T fragments stay in
//                                                    registers for the whole unit)
//   O^T[D x 8]        += V^T[D x 16] . P^T[16 x 8]   (P^T fragments come from the S^T
//                                                    accumulators by one movmatrix
//                                                    transpose per 8x8 half)
//
// K/V stages arrive through TMA tensor-map loads with the 128-byte swizzle (two 64-column
// boxes per D=128 row), which makes every ldmatrix conflict-free.  Softmax statistics stay in
// fp32 (online max / sum, base-2 exponent); P is rounded to the K/V type for the P.V tile,
// the accumulators are fp32.
#pragma once
#include <cuda.h>

#include <type_traits>

#include "attn_decode.cuh"

// Launch shape of the tensor-core decode kernel: 2 warps x 2 stages per CTA measured best
// (or tied) on every workload; overridable at build time for tuning sweeps.
#ifndef PKV_DECODE_TC_WARPS
#define PKV_DECODE_TC_WARPS 2
#endif
#ifndef PKV_DECODE_TC_STAGES
#define PKV_DECODE_TC_STAGES 2
#endif
// 1: the softmax weights are computed before the rescale vote resolves, as in the FP8
// decode (the same bits either way; measured +1.4 / +1.7 % on the fork / beam steps, within
// noise elsewhere).
#ifndef PKV_TC_SPEC_EXP
#define PKV_TC_SPEC_EXP 1
#endif

namespace pkv {

template <typename T, int D, int G, int W, int NSW>
struct DecodeTcCfg {
    static constexpr int CHUNK = kBlock * D * 2;   // bytes of one (block, kv head) of K or V
    static constexpr int HALVES = D * 2 / 128;     // 128-byte swizzle boxes per token row
    static constexpr int BOX = kBlock * 128;       // bytes of one box (16 rows x 128 B)
    static constexpr int STAGE = 2 * CHUNK;        // K chunk then V chunk
    static constexpr int RING = W * NSW * STAGE;
    static constexpr int BARS = W * NSW * 8;
    static constexpr int MRG = W * G * (D + 2) * 4;
    static constexpr int SMEM = 1024 + RING + BARS + MRG;  // + slack to align the ring
    static constexpr int KSTEPS = D / 16;
    static_assert(D == 64 || D == 128, "head_dim 64 or 128");
    static_assert(G <= 8, "at most 8 query heads per kv head (one n=8 tile)");
};

// The work of one CTA.  kContig false: the paged pools, block j of sequence s at physical
// block block_tables[s][j], TMA row (phys * H_kv + hk) * 16.  kContig true: a contiguous cache
// [S][H_kv][Lmax][D] with no block table, block j of sequence s at TMA row
// (s * H_kv + hk) * Lmax + 16 j; everything else is the same code.
template <typename T, int D, int G, int W, int NSW, bool kContig>
__device__ __forceinline__ void decode_tc_body(const CUtensorMap &tmk, const CUtensorMap &tmv,
                                               const DecodeParams &p) {
    using C = DecodeTcCfg<T, D, G, W, NSW>;
    constexpr bool BF = std::is_same<T, __nv_bfloat16>::value;
    constexpr int CHUNK = C::CHUNK, KSTEPS = C::KSTEPS, HALVES = C::HALVES, BOX = C::BOX;
    constexpr unsigned FULL = 0xffffffffu;

    extern __shared__ unsigned char smem_raw[];
    unsigned char *smem = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

    pdl_launch_dependents();

    const int bid = blockIdx.x;
    const int part = bid % p.pmax;
    const int rest = bid / p.pmax;
    const int hk = rest % p.Hkv;
    const int s = rest / p.Hkv;

    const int L = p.context_lens[s];
    if (L < 1 || L > (p.maxB << p.bshift)) {
        if (part == 0 && hk == 0 && threadIdx.x == 0) atomicOr(&g_faults, kFaultBadLen);
        return;
    }
    const int nblk = (L + kBlock - 1) / kBlock;
    const int nparts = (nblk + p.part_blocks - 1) / p.part_blocks;
    if (part >= nparts) return;
    const int j0 = part * p.part_blocks;
    const int nb = min(nblk, j0 + p.part_blocks) - j0;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int g = lane >> 2;   // fragment row group
    const int tq = lane & 3;   // fragment column pair
    const int nbw = nb > warp ? (nb - warp + W - 1) / W : 0;

    unsigned char *ring = smem + warp * NSW * C::STAGE;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::RING) + warp * NSW;
    float *mo = reinterpret_cast<float *>(smem + C::RING + C::BARS);  // [W][G][D]
    float *mml = mo + W * G * D;                                      // [W][G][2]

    if (lane == 0) {
#pragma unroll
        for (int i = 0; i < NSW; ++i) mbar_init(&bars[i], 1);
        fence_mbar_init();
        if (warp == 0) {
            prefetch_tmap(&tmk);
            prefetch_tmap(&tmv);
        }
    }
    __syncwarp();
    if (!kContig && p.slot_mapping != nullptr && part == nparts - 1 && warp == (nb - 1) % W)
        write_newest_token<T, D>(p, s, hk, L, lane);

    const int32_t *btab = kContig ? nullptr : p.block_tables + (size_t)s * p.maxB;
    const int j1 = j0 + warp;  // this warp's first sub-block
    const uint64_t policy = l2_evict_first_policy();
    int tab_chunk = 0;
    int32_t tab = !kContig && lane < nbw ? btab[sub_to_entry(j1 + W * lane, p.bshift)] : 0;
    // contiguous cache: TMA row of this warp's first block
    const int32_t crow0 = kContig ? (s * p.Hkv + hk) * p.Lmax + (j0 + warp) * kBlock : 0;

    // Issue block i of this warp into stage i % NSW: HALVES boxes of K, then of V.
    auto issue = [&](int i) {
        int32_t phys = 0;
        if constexpr (!kContig) {
            if ((i >> 5) != tab_chunk) {
                tab_chunk = i >> 5;
                const int li = (tab_chunk << 5) + lane;
                tab = li < nbw ? btab[sub_to_entry(j1 + W * li, p.bshift)] : 0;
            }
            phys = __shfl_sync(FULL, tab, i & 31);
        }
        if (lane == 0 && !withheld_for_test(i, warp)) {
            uint64_t *bar = &bars[i % NSW];
            unsigned char *dst = ring + (i % NSW) * C::STAGE;
            if (kContig || (unsigned)phys < (unsigned)p.NB) {
                const int32_t row = kContig ? crow0 + i * (W * kBlock)
                                            : ((phys * p.Hkv + hk) << p.bshift) +
                                                  sub_row(j1 + W * i, p.bshift);
                fence_proxy_async_smem();
                mbar_arrive_expect_tx(bar, 2 * CHUNK);
#pragma unroll
                for (int h = 0; h < HALVES; ++h) {
                    tma_load_2d(dst + h * BOX, &tmk, h * 64, row, bar, policy);
                    tma_load_2d(dst + CHUNK + h * BOX, &tmv, h * 64, row, bar, policy);
                }
            } else {
                atomicOr(&g_faults, kFaultBadBlock);
                mbar_arrive(bar);
            }
        }
    };

    const int npro = nbw < NSW ? nbw : NSW;
    for (int i = 0; i < npro; ++i) issue(i);
    int issued = npro;

    // Q^T as the B operand of S^T = K Q^T: lane (g, tq) holds head g, dims 16j+2tq(+1) and
    // 16j+2tq+8(+9); heads g >= G are zero columns.
    uint32_t qb[KSTEPS][2];
    {
        const bool hv = g < G;
        const uint32_t *qrow = reinterpret_cast<const uint32_t *>(
            static_cast<const T *>(p.q) + ((size_t)s * p.Hq + hk * G + (hv ? g : 0)) * D);
#pragma unroll
        for (int j = 0; j < KSTEPS; ++j) {
            qb[j][0] = hv ? qrow[8 * j + tq] : 0u;
            qb[j][1] = hv ? qrow[8 * j + tq + 4] : 0u;
        }
    }

    float o[KSTEPS][4];  // O^T m-tiles over the head dimension
#pragma unroll
    for (int i = 0; i < KSTEPS; ++i)
#pragma unroll
        for (int e = 0; e < 4; ++e) o[i][e] = 0.f;
    float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
    const float sl = p.scale_log2;

    // ldmatrix row roles: K (A of S^T, plain) and V (A of O^T, transposed)
    const int k_tok = (lane & 7) + 8 * ((lane >> 3) & 1);
    const int k_c = lane >> 4;
    const int v_tok = (lane & 7) + 8 * (lane >> 4);
    const int v_c = (lane >> 3) & 1;

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
            // V rows past the context may hold anything (even NaN): zero them so that the
            // P.V tile, whose P is 0 there, cannot pick them up.
            constexpr int UNITS = HALVES * 8;  // 16-byte units per row
            for (int u = lane; u < (kBlock - nvalid) * UNITS; u += 32) {
                const int r = nvalid + u / UNITS;
                const int h = (u % UNITS) / 8, cc = u % 8;
                *reinterpret_cast<uint4 *>(Vs + h * BOX + r * 128 + cc * 16) =
                    make_uint4(0u, 0u, 0u, 0u);
            }
            fence_proxy_async_smem();
            __syncwarp();
        }

        // ---- S^T = K Q^T ---------------------------------------------------------------
        float sacc[4] = {0.f, 0.f, 0.f, 0.f};
        const uint32_t kb = smem_u32(Ks);
#pragma unroll
        for (int j = 0; j < KSTEPS; ++j) {
            const int c = 2 * j + k_c;
            const uint32_t addr = kb + (c >> 3) * BOX + k_tok * 128 +
                                  ((((c & 7) ^ (k_tok & 7))) << 4);
            uint32_t a[4];
            ldmatrix_x4(a, addr);
            mma_16816<BF>(sacc, a, qb[j][0], qb[j][1]);
        }

        // ---- online softmax: lane holds tokens g, g+8 of heads 2tq, 2tq+1 ------------
        float x0 = sacc[0] * sl, x1 = sacc[1] * sl, x2 = sacc[2] * sl, x3 = sacc[3] * sl;
        if (nvalid < kBlock) {  // the sequence's last block: no weight past its end
            x0 = g < nvalid ? x0 : -INFINITY;
            x1 = g < nvalid ? x1 : -INFINITY;
            x2 = g + 8 < nvalid ? x2 : -INFINITY;
            x3 = g + 8 < nvalid ? x3 : -INFINITY;
        }
        // Lazy rescale: a head's reference max moves only when a block's max passes it by
        // more than kLazyRescale (base 2), so P stays <= 2^kLazyRescale; O / l does not
        // depend on the reference.  One vote tells whether any score passes its reference
        // by that much; only then (a warp's first block, and rarely after) does the warp
        // reduce the block's max and rescale O and its partial sums.
#if PKV_TC_SPEC_EXP
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
#if PKV_TC_SPEC_EXP
            p0 = ex2_ftz(x0 - m_run[0]);
            p1 = ex2_ftz(x1 - m_run[1]);
            p2 = ex2_ftz(x2 - m_run[0]);
            p3 = ex2_ftz(x3 - m_run[1]);
#endif
        }
#if !PKV_TC_SPEC_EXP
        const float p0 = ex2_ftz(x0 - m_run[0]), p1 = ex2_ftz(x1 - m_run[1]);
        const float p2 = ex2_ftz(x2 - m_run[0]), p3 = ex2_ftz(x3 - m_run[1]);
#endif
        // per-lane partial sums; the 8 token-row lanes of a head add theirs after the loop
        l_run[0] += p0 + p2;
        l_run[1] += p1 + p3;

        // P^T fragments (k = token, n = head) by transposing the two 8x8 halves of P
        const uint32_t b0 = movmatrix_trans(pack2<BF>(p0, p1));
        const uint32_t b1 = movmatrix_trans(pack2<BF>(p2, p3));

        // ---- O^T += V^T P^T ------------------------------------------------------------
        const uint32_t vb = smem_u32(Vs);
#pragma unroll
        for (int t = 0; t < KSTEPS; ++t) {
            const int c = 2 * t + v_c;
            const uint32_t addr = vb + (c >> 3) * BOX + v_tok * 128 +
                                  ((((c & 7) ^ (v_tok & 7))) << 4);
            uint32_t a[4];
            ldmatrix_x4_trans(a, addr);
            mma_16816<BF>(o[t], a, b0, b1);
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

    // ---- warp state -> shared memory; heads 2tq and 2tq+1 of this lane ----------------
    const int h0 = 2 * tq, h1 = 2 * tq + 1;
    if (h0 < G) {
        float *dst = mo + (warp * G + h0) * D;
#pragma unroll
        for (int t = 0; t < KSTEPS; ++t) {
            dst[16 * t + g] = o[t][0];
            dst[16 * t + g + 8] = o[t][2];
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
            dst[16 * t + g] = o[t][1];
            dst[16 * t + g + 8] = o[t][3];
        }
        if (g == 0) {
            mml[(warp * G + h1) * 2] = m_run[1];
            mml[(warp * G + h1) * 2 + 1] = l_run[1];
        }
    }
    __syncthreads();
    merge_and_store<T, D, G, W>(p, mo, mml, s, hk, part, nparts);
}

template <typename T, int D, int G, int W, int NSW>
__global__ void __launch_bounds__(W * 32)
paged_attn_decode_tc_kernel(const __grid_constant__ CUtensorMap tmk,
                            const __grid_constant__ CUtensorMap tmv, const DecodeParams p) {
    decode_tc_body<T, D, G, W, NSW, false>(tmk, tmv, p);
}

// The same decode over a contiguous cache (no block table): the comparison kernel for the
// cost of the table's indirection.
template <typename T, int D, int G, int W, int NSW>
__global__ void __launch_bounds__(W * 32)
contiguous_attn_decode_tc_kernel(const __grid_constant__ CUtensorMap tmk,
                                 const __grid_constant__ CUtensorMap tmv, const DecodeParams p) {
    decode_tc_body<T, D, G, W, NSW, true>(tmk, tmv, p);
}

}  // namespace pkv
