// Paged decode attention for sm_100a.
//
// What it computes ("Memory Optimization in LLM Serving with PagedAttention", section "How
// PagedAttention Works": a custom kernel gathers the scattered KV blocks through the block
// table to compute attention): for each sequence s and query head h, softmax(q K^T * scale) V
// over the sequence's context_lens[s] cached tokens, K/V rows fetched from the physical block
// block_tables[s][t / 16], offset t % 16.
//
// How (B200 design):
//   * one CTA per work unit (sequence, kv head, context partition); the CTA serves all
//     H_q/H_kv query heads that share the kv head, so each K/V block is read from HBM once;
//   * W consumer warps; warp w takes the unit's blocks w, w+W, w+2W, ...; each warp owns a
//     ring of NSW shared-memory stages and keeps it full with the bulk async copy engine
//     (one elected lane issues two contiguous 16*D-element copies, K and V, per block,
//     completion counted in bytes on the stage's mbarrier, bounded waits);
//   * per 16-token block: lane (c, r) owns 16-byte chunk c of the head dimension and tokens
//     r, r+TPP, ...; it forms partial q.k sums from conflict-free 16-byte shared loads, a
//     shuffle reduce-scatter finishes the dot products, then an online softmax (running
//     max / sum, fp32, base-2 exponent with scale*log2(e) folded into q) and the P.V update;
//   * at the end the W warps' (max, sum, unnormalised output) states are merged in shared
//     memory; a unit covering the whole sequence writes the normalised output, otherwise it
//     writes its partial state for the log-sum-exp reduce kernel below.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstdint>
#include <type_traits>

#include "faults.cuh"
#include "ptx.cuh"

namespace pkv {

// Launch shape of the CUDA-core decode kernel (consumer warps per CTA, stages per warp) and
// the default context partition; overridable at build time for tuning sweeps.
#ifndef PKV_DECODE_WARPS
#define PKV_DECODE_WARPS 4
#endif
#ifndef PKV_DECODE_STAGES
#define PKV_DECODE_STAGES 2
#endif
constexpr int kDefaultPartitionTokens = 512;

// Tokens per KV sub-block: the unit every kernel stages and multiplies (one TMA box, one MMA
// tile).  A physical block holds 16 or 32 tokens (1 << DecodeParams::bshift): sub-block j of
// a sequence is rows 16 * (j mod (B / 16)) .. of physical block block_tables[s][j / (B / 16)].
constexpr int kBlock = 16;
// Lazy online-softmax rescale threshold (base-2 logit units): a running max moves only when
// a block's max exceeds it by more than this, so exponents stay <= 2^8.
#ifndef PKV_LAZY_RESCALE
#define PKV_LAZY_RESCALE 8
#endif
constexpr float kLazyRescale = float(PKV_LAZY_RESCALE);
// Bounded shared-memory barrier waits give up after this long (1 s; test builds shorten it).
#ifndef PKV_WAIT_TIMEOUT_NS
#define PKV_WAIT_TIMEOUT_NS 1000000000ull
#endif
constexpr uint64_t kWaitTimeoutNs = PKV_WAIT_TIMEOUT_NS;

// Test builds only (-DPKV_TEST_WITHHOLD_BLOCK=i): warp 0 of the grid's first CTA issues
// neither the copy nor the arrival of its i-th block, so its bounded wait on that stage runs
// out and the timeout path runs (fault bit, drain of the copies still in flight, an empty
// state for the warp).  No copy targets the withheld stage, so nothing is left in flight.
__device__ __forceinline__ bool withheld_for_test(int i, int warp) {
#ifdef PKV_TEST_WITHHOLD_BLOCK
    return blockIdx.x == 0 && warp == 0 && i == PKV_TEST_WITHHOLD_BLOCK;
#else
    (void)i;
    (void)warp;
    return false;
#endif
}


struct DecodeParams {
    const void *q;
    const void *k_pool;
    const void *v_pool;
    const int32_t *block_tables;
    const int32_t *context_lens;
    void *out;
    float *ws_o;   // [S][H_q][pmax][D] unnormalised partition outputs (split only)
    float *ws_ml;  // [S][H_q][pmax][2]  partition (max, sum), base-2 units (split only)
    int32_t S, Hq, Hkv, NB, maxB;
    int32_t part_blocks;  // blocks per partition
    int32_t pmax;         // partitions of the longest admissible sequence
    float scale_log2;     // scale * log2(e)
    // fused kv_write (NULL: none): token s of k_new / v_new [S][H_kv][D] is sequence s's
    // newest token, stored into slot_mapping[s] before the decode reads it
    const void *k_new = nullptr;
    const void *v_new = nullptr;
    const int64_t *slot_mapping = nullptr;
    // contiguous cache (attn_decode_contiguous): token rows per (sequence, kv head); 0 for
    // the paged pools
    int32_t Lmax = 0;
    // log2 of the tokens per physical block (4: 16-token blocks, 5: 32-token blocks)
    int32_t bshift = 4;
};

// Table entry of sub-block j (of kBlock tokens) and the sub-block's first row within its
// physical block: sub-block j lies in table entry j >> (bshift - 4), at row 16 * (j & ...).
__device__ __forceinline__ int sub_to_entry(int j, int bshift) { return j >> (bshift - 4); }
__device__ __forceinline__ int sub_row(int j, int bshift) {
    return (j & ((1 << (bshift - 4)) - 1)) * kBlock;
}

// Fused kv_write, called by the one warp per (sequence, kv head) that will copy the block
// holding position L-1.  The warp stores the newest token's K and V rows of kv head hk into
// their slot, then fences its generic-proxy stores against its own later bulk / TMA copies
// (async proxy) of that block.  A slot of -1 is skipped; a slot other than the one of
// position L-1 is not written and sets fault bit 4 (bad slot).
template <typename T, int D>
__device__ __forceinline__ void write_newest_token(const DecodeParams &p, int s, int hk, int L,
                                                   int lane) {
    const int64_t slot = p.slot_mapping[s];
    if (slot != -1) {
        const int32_t blk = p.block_tables[(size_t)s * p.maxB + ((L - 1) >> p.bshift)];
        const int off = (L - 1) & ((1 << p.bshift) - 1);
        if ((unsigned)blk < (unsigned)p.NB && slot == ((int64_t)blk << p.bshift) + off) {
            constexpr int VPR = D * (int)sizeof(T) / 16;  // 16-byte vectors per row
            const size_t src = ((size_t)s * p.Hkv + hk) * VPR;
            const size_t dst = ((((size_t)blk * p.Hkv + hk) << p.bshift) + off) * VPR;
            // the pools are written only here; the decode itself reads them
            uint4 *kp = static_cast<uint4 *>(const_cast<void *>(p.k_pool));
            uint4 *vp = static_cast<uint4 *>(const_cast<void *>(p.v_pool));
            for (int v = lane; v < 2 * VPR; v += 32) {
                if (v < VPR)
                    kp[dst + v] = static_cast<const uint4 *>(p.k_new)[src + v];
                else
                    vp[dst + v - VPR] = static_cast<const uint4 *>(p.v_new)[src + v - VPR];
            }
            fence_proxy_async_global();
        } else if (lane == 0) {
            atomicOr(&g_faults,
                     (unsigned)blk < (unsigned)p.NB ? kFaultBadSlot : kFaultBadBlock);
        }
    }
    __syncwarp();
}

// ---- element conversions --------------------------------------------------------------
template <typename T>
struct Elem;

template <>
struct Elem<float> {
    static constexpr int kPer16B = 4;
    __device__ static __forceinline__ void load(const uint4 &v, float (&f)[4]) {
        f[0] = __uint_as_float(v.x);
        f[1] = __uint_as_float(v.y);
        f[2] = __uint_as_float(v.z);
        f[3] = __uint_as_float(v.w);
    }
    __device__ static __forceinline__ float from_float(float x) { return x; }
};

template <>
struct Elem<__half> {
    static constexpr int kPer16B = 8;
    __device__ static __forceinline__ void load(const uint4 &v, float (&f)[8]) {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            __half2 h = *reinterpret_cast<const __half2 *>(&w[i]);
            float2 a = __half22float2(h);
            f[2 * i] = a.x;
            f[2 * i + 1] = a.y;
        }
    }
    __device__ static __forceinline__ __half from_float(float x) { return __float2half_rn(x); }
};

template <>
struct Elem<__nv_bfloat16> {
    static constexpr int kPer16B = 8;
    // bfloat16 is the upper half of a binary32: widening is a shift / mask.
    __device__ static __forceinline__ void load(const uint4 &v, float (&f)[8]) {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[2 * i] = __uint_as_float(w[i] << 16);
            f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
    __device__ static __forceinline__ __nv_bfloat16 from_float(float x) {
        return __float2bfloat16_rn(x);
    }
};

// Store E floats as E elements of T (16 bytes for 16-bit T, 16 bytes for float).
template <typename T, int E>
__device__ __forceinline__ void store_row(T *dst, const float (&x)[E]) {
    static_assert(E * sizeof(T) == 16, "one 16-byte vector");
    union {
        uint4 v;
        T e[E];
    } u;
#pragma unroll
    for (int i = 0; i < E; ++i) u.e[i] = Elem<T>::from_float(x[i]);
    *reinterpret_cast<uint4 *>(dst) = u.v;
}

// Load G consecutive floats from shared memory (vectorised; p is 4*G-byte aligned).
template <int G>
__device__ __forceinline__ void load_g(const float *p, float (&x)[G]) {
    if constexpr (G % 4 == 0) {
#pragma unroll
        for (int i = 0; i < G; i += 4) {
            const float4 v = *reinterpret_cast<const float4 *>(p + i);
            x[i] = v.x;
            x[i + 1] = v.y;
            x[i + 2] = v.z;
            x[i + 3] = v.w;
        }
    } else if constexpr (G == 2) {
        const float2 v = *reinterpret_cast<const float2 *>(p);
        x[0] = v.x;
        x[1] = v.y;
    } else {
#pragma unroll
        for (int i = 0; i < G; ++i) x[i] = p[i];
    }
}

// Merge the W warps' (max, sum, unnormalised output) states of one work unit from shared
// memory (mo [W][G][D], mml [W][G][2], base-2 units) and write either the normalised output
// (the unit covers the whole sequence) or the unit's partial state for the reduce kernel.
// Called by all W*32 threads after a __syncthreads().
template <typename T, int D, int G, int W>
__device__ __forceinline__ void merge_and_store(const DecodeParams &p, const float *mo,
                                                const float *mml, int s, int hk, int part,
                                                int nparts) {
    constexpr int E = 16 / sizeof(T);
    constexpr int VPH = D / E;  // 16-byte output vectors per head
    for (int idx = threadIdx.x; idx < G * VPH; idx += W * 32) {
        const int hh = idx / VPH;
        const int d0 = (idx % VPH) * E;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < W; ++w) M = fmaxf(M, mml[(w * G + hh) * 2]);
        float den = 0.f, num[E];
#pragma unroll
        for (int e = 0; e < E; ++e) num[e] = 0.f;
#pragma unroll
        for (int w = 0; w < W; ++w) {
            const float mw = mml[(w * G + hh) * 2];
            const float a = mw == -INFINITY ? 0.f : exp2f(mw - M);
            den += a * mml[(w * G + hh) * 2 + 1];
#pragma unroll
            for (int e = 0; e < E; ++e) num[e] += a * mo[(w * G + hh) * D + d0 + e];
        }
        const int h = hk * G + hh;
        if (nparts == 1) {
            const float inv = 1.f / den;
#pragma unroll
            for (int e = 0; e < E; ++e) num[e] *= inv;
            store_row<T, E>(static_cast<T *>(p.out) + ((size_t)s * p.Hq + h) * D + d0, num);
        } else {
            const size_t row = ((size_t)s * p.Hq + h) * p.pmax + part;
            float4 *dst = reinterpret_cast<float4 *>(p.ws_o + row * D + d0);
#pragma unroll
            for (int e = 0; e < E; e += 4)
                dst[e / 4] = make_float4(num[e], num[e + 1], num[e + 2], num[e + 3]);
            if (d0 == 0) {
                p.ws_ml[row * 2] = M;
                p.ws_ml[row * 2 + 1] = den;
            }
        }
    }
}

template <typename T, int D, int G, int W, int NSW>
struct DecodeCfg {
    static constexpr int ES = sizeof(T);
    static constexpr int E = 16 / ES;             // elements per 16-byte chunk
    static constexpr int CPR = D * ES / 16;       // chunks per token row
    static constexpr int TPP = 32 / CPR;          // tokens per pass of the warp
    static constexpr int NPASS = kBlock / TPP;    // passes per block
    static constexpr int NV = NPASS * G;          // partial scores per lane
    static constexpr int HG = G >= 2 ? G / 2 : 1; // heads per lane after the reduction
    static constexpr int NE = G >= 2 ? G / 2 : 1; // softmax entries per lane
    static constexpr int CHUNK = kBlock * D * ES; // bytes of one (block, kv head)
    static constexpr int RING = W * NSW * 2 * CHUNK;
    static constexpr int BARS = W * NSW * 8;
    static constexpr int SCR = W * (kBlock * G + G) * 4;   // per-warp scores / rescale
    static constexpr int MRG = W * G * (D + 2) * 4;        // cross-warp merge
    static constexpr int SMEM = RING + BARS + SCR + MRG;
    static_assert(CPR >= 8 && CPR <= 32, "head_dim * elem_size must be 128..512 bytes");
    static_assert(NV <= 64, "too many partial scores per lane");
};

template <typename T, int D, int G, int W, int NSW>
__global__ void __launch_bounds__(W * 32)
paged_attn_decode_kernel(const DecodeParams p) {
    using C = DecodeCfg<T, D, G, W, NSW>;
    constexpr int E = C::E, CPR = C::CPR, TPP = C::TPP, NPASS = C::NPASS, NV = C::NV;
    constexpr int HG = C::HG, NE = C::NE, CHUNK = C::CHUNK;
    constexpr unsigned FULL = 0xffffffffu;

    extern __shared__ __align__(128) unsigned char smem[];

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
    const int c = lane % CPR;   // 16-byte chunk of the head dimension
    const int r = lane / CPR;   // token phase within a pass
    const int nbw = nb > warp ? (nb - warp + W - 1) / W : 0;

    unsigned char *ring = smem + warp * NSW * 2 * CHUNK;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::RING) + warp * NSW;
    float *sc = reinterpret_cast<float *>(smem + C::RING + C::BARS) + warp * (kBlock * G + G);
    float *al = sc + kBlock * G;
    float *mo = reinterpret_cast<float *>(smem + C::RING + C::BARS + C::SCR);  // [W][G][D]
    float *mml = mo + W * G * D;                                               // [W][G][2]

    if (lane == 0) {
#pragma unroll
        for (int i = 0; i < NSW; ++i) mbar_init(&bars[i], 1);
        fence_mbar_init();
    }
    __syncwarp();
    if (p.slot_mapping != nullptr && part == nparts - 1 && warp == (nb - 1) % W)
        write_newest_token<T, D>(p, s, hk, L, lane);

    const int32_t *btab = p.block_tables + (size_t)s * p.maxB;
    const int j1 = j0 + warp;  // this warp's first sub-block
    const char *kbase = static_cast<const char *>(p.k_pool);
    const char *vbase = static_cast<const char *>(p.v_pool);
    const uint64_t policy = l2_evict_first_policy();

    // Block-table entries of this warp's sub-blocks, 32 at a time (lane i holds sub-block i).
    int tab_chunk = 0;
    int32_t tab = lane < nbw ? btab[sub_to_entry(j1 + W * lane, p.bshift)] : 0;

    // Issue sub-block i of this warp into stage i % NSW (all lanes call; lane 0 issues).
    auto issue = [&](int i) {
        if ((i >> 5) != tab_chunk) {
            tab_chunk = i >> 5;
            const int li = (tab_chunk << 5) + lane;
            tab = li < nbw ? btab[sub_to_entry(j1 + W * li, p.bshift)] : 0;
        }
        const int32_t phys = __shfl_sync(FULL, tab, i & 31);
        if (lane == 0 && !withheld_for_test(i, warp)) {
            uint64_t *bar = &bars[i % NSW];
            unsigned char *dst = ring + (i % NSW) * 2 * CHUNK;
            if ((unsigned)phys < (unsigned)p.NB) {
                const size_t row = (((size_t)phys * p.Hkv + hk) << p.bshift) +
                                   (size_t)sub_row(j1 + W * i, p.bshift);
                const size_t off = row * (size_t)(CHUNK / kBlock);
                fence_proxy_async_smem();
                mbar_arrive_expect_tx(bar, 2 * CHUNK);
                bulk_g2s(dst, kbase + off, CHUNK, bar, policy);
                bulk_g2s(dst + CHUNK, vbase + off, CHUNK, bar, policy);
            } else {
                atomicOr(&g_faults, kFaultBadBlock);
                mbar_arrive(bar);  // complete the phase without data
            }
        }
    };

    const int npro = nbw < NSW ? nbw : NSW;
    for (int i = 0; i < npro; ++i) issue(i);
    int issued = npro;

    // Query rows of the group, pre-scaled into base-2 logits.
    float q[G][E];
#pragma unroll
    for (int hh = 0; hh < G; ++hh) {
        const T *qrow = static_cast<const T *>(p.q) + ((size_t)s * p.Hq + hk * G + hh) * D;
        const uint4 v = *reinterpret_cast<const uint4 *>(qrow + c * E);
        Elem<T>::load(v, q[hh]);
#pragma unroll
        for (int e = 0; e < E; ++e) q[hh][e] *= p.scale_log2;
    }

    float o[G][E];
#pragma unroll
    for (int hh = 0; hh < G; ++hh)
#pragma unroll
        for (int e = 0; e < E; ++e) o[hh][e] = 0.f;
    float m_run[NE], l_run[NE];
#pragma unroll
    for (int k = 0; k < NE; ++k) {
        m_run[k] = -INFINITY;
        l_run[k] = 0.f;
    }

    bool dead = false;
    int i = 0;
    for (; i < nbw; ++i) {
        const int st = i % NSW;
        if (!mbar_wait_bounded(&bars[st], (uint32_t)(i / NSW) & 1u, kWaitTimeoutNs)) {
            if (lane == 0) atomicOr(&g_faults, kFaultTimeout);
            dead = true;
            break;
        }
        const unsigned char *Ks = ring + st * 2 * CHUNK;
        const unsigned char *Vs = Ks + CHUNK;
        const int jb = j0 + warp + W * i;                // logical block
        const int nvalid = min(kBlock, L - jb * kBlock); // tokens of this block in context

        // ---- partial scores: v[ii * G + hh] over this lane's chunk -------------------
        float v[NV];
#pragma unroll
        for (int ii = 0; ii < NPASS; ++ii) {
            const int t = r + TPP * ii;
            const uint4 kv = *reinterpret_cast<const uint4 *>(Ks + (t * CPR + c) * 16);
            float kf[E];
            Elem<T>::load(kv, kf);
#pragma unroll
            for (int hh = 0; hh < G; ++hh) {
                float a = q[hh][0] * kf[0];
#pragma unroll
                for (int e = 1; e < E; ++e) a = fmaf(q[hh][e], kf[e], a);
                v[ii * G + hh] = a;
            }
        }
        // ---- reduce-scatter over the CPR lanes sharing a token phase ----------------
        int n = NV;
#pragma unroll
        for (int m = CPR / 2; m >= 1; m >>= 1) {
            if (n > 1) {
                const bool up = (lane & m) != 0;
                const int half = n / 2;
#pragma unroll
                for (int j = 0; j < NV / 2; ++j) {
                    if (j < half) {
                        const float send = up ? v[j] : v[j + half];
                        const float keep = up ? v[j + half] : v[j];
                        v[j] = keep + __shfl_xor_sync(FULL, send, m);
                    }
                }
                n = half;
            } else {
                v[0] += __shfl_xor_sync(FULL, v[0], m);
            }
        }
        // lane now holds the logits of token tt for heads hh0 .. hh0+HG-1
        {
            const int tt = r + TPP * (c >> 1);
            const int hh0 = G >= 2 ? (c & 1) * HG : 0;
#pragma unroll
            for (int k = 0; k < HG; ++k) sc[tt * G + hh0 + k] = tt < nvalid ? v[k] : -INFINITY;
        }
        __syncwarp();

        // ---- online softmax over the block: entry (head hh, token lane % 16) --------
#pragma unroll
        for (int k = 0; k < NE; ++k) {
            const int hh = G >= 2 ? (lane >> 4) + 2 * k : 0;
            const int tt = lane & 15;
            const float x = sc[tt * G + hh];
            float bm = x;
#pragma unroll
            for (int m = 1; m < 16; m <<= 1) bm = fmaxf(bm, __shfl_xor_sync(FULL, bm, m));
            const float mn = fmaxf(m_run[k], bm);
            const float pv = exp2f(x - mn);
            float sum = pv;
#pragma unroll
            for (int m = 1; m < 16; m <<= 1) sum += __shfl_xor_sync(FULL, sum, m);
            const float a = exp2f(m_run[k] - mn);
            l_run[k] = l_run[k] * a + sum;
            m_run[k] = mn;
            sc[tt * G + hh] = pv;
            if (tt == 0) al[hh] = a;
        }
        __syncwarp();

        // ---- P.V ----------------------------------------------------------------------
        {
            float alv[G];
            load_g<G>(al, alv);
#pragma unroll
            for (int hh = 0; hh < G; ++hh)
#pragma unroll
                for (int e = 0; e < E; ++e) o[hh][e] *= alv[hh];
        }
#pragma unroll
        for (int ii = 0; ii < NPASS; ++ii) {
            const int t = r + TPP * ii;
            if (t < nvalid) {
                const uint4 vv = *reinterpret_cast<const uint4 *>(Vs + (t * CPR + c) * 16);
                float vf[E];
                Elem<T>::load(vv, vf);
                float pr[G];
                load_g<G>(sc + t * G, pr);
#pragma unroll
                for (int hh = 0; hh < G; ++hh)
#pragma unroll
                    for (int e = 0; e < E; ++e) o[hh][e] = fmaf(pr[hh], vf[e], o[hh][e]);
            }
        }
        __syncwarp();

        if (issued < nbw) {
            issue(issued);
            ++issued;
        }
    }
    if (dead) {
        // Let copies still in flight (blocks i .. issued-1, at most one per stage) land
        // before the CTA retires; bounded as well.
        for (int b = i; b < issued; ++b) {
            (void)mbar_wait_bounded(&bars[b % NSW], (uint32_t)(b / NSW) & 1u, kWaitTimeoutNs);
        }
#pragma unroll
        for (int k = 0; k < NE; ++k) {
            m_run[k] = -INFINITY;
            l_run[k] = 0.f;
        }
#pragma unroll
        for (int hh = 0; hh < G; ++hh)
#pragma unroll
            for (int e = 0; e < E; ++e) o[hh][e] = 0.f;
    }

    // ---- warp state -> shared memory ---------------------------------------------------
#pragma unroll
    for (int m = CPR; m < 32; m <<= 1)
#pragma unroll
        for (int hh = 0; hh < G; ++hh)
#pragma unroll
            for (int e = 0; e < E; ++e) o[hh][e] += __shfl_xor_sync(FULL, o[hh][e], m);
    if (lane < CPR) {
#pragma unroll
        for (int hh = 0; hh < G; ++hh)
#pragma unroll
            for (int e = 0; e < E; ++e) mo[(warp * G + hh) * D + c * E + e] = o[hh][e];
    }
    if ((lane & 15) == 0) {
#pragma unroll
        for (int k = 0; k < NE; ++k) {
            const int hh = G >= 2 ? (lane >> 4) + 2 * k : 0;
            mml[(warp * G + hh) * 2 + 0] = m_run[k];
            mml[(warp * G + hh) * 2 + 1] = l_run[k];
        }
    }
    __syncthreads();

    merge_and_store<T, D, G, W>(p, mo, mml, s, hk, part, nparts);
}

// ---- log-sum-exp merge of the partitions of split sequences ----------------------------
// out[s,h,:] = sum_p 2^(m_p - M) o_p / sum_p 2^(m_p - M) l_p,  M = max_p m_p  (base-2 units,
// which is the natural-log formula with every logit scaled by log2(e)).  The kernel reads a
// few KB a row from L2 right after the decode wrote them, so its time is round trips, and it
// is built to take as few as possible:
//   * R warps per (sequence, query head) row: one when no row has more than kReduceBatch
//     partitions (four rows to a CTA), else kReduceWideWarps (one row to a CTA);
//   * warp w of a row takes partitions w, w+R, w+2R, ... in batches of kReduceBatch whose
//     (m, l) pairs and o_p slices (a D/32-float slice per lane) are all loaded before the
//     first is used, so a row of up to R * kReduceBatch partitions costs one round trip;
//   * each warp keeps its own running max (rescaling its sums when a batch raises it), and
//     with R > 1 the warps' states meet in shared memory under the same merge formula.
// A partition whose m is -inf (no state) weighs 0; a row with no state at all comes out NaN.
// Rows whose sequence fits in one partition were already written by the decode kernel.
constexpr int kReduceBatch = 8;
constexpr int kReduceWideWarps = 8;

template <int VL>
struct ReduceVec;
template <>
struct ReduceVec<2> {
    using type = float2;
    __device__ static float get(const float2 &v, int k) { return k == 0 ? v.x : v.y; }
};
template <>
struct ReduceVec<4> {
    using type = float4;
    __device__ static float get(const float4 &v, int k) {
        return k == 0 ? v.x : k == 1 ? v.y : k == 2 ? v.z : v.w;
    }
};

// N floats to N consecutive elements of T (one 4-, 8- or 16-byte store).
template <typename T, int N>
__device__ __forceinline__ void store_vec(T *dst, const float (&x)[N]) {
    constexpr int kBytes = N * (int)sizeof(T);
    static_assert(kBytes == 4 || kBytes == 8 || kBytes == 16, "one 4/8/16-byte vector");
    using V = typename std::conditional<
        kBytes == 16, uint4, typename std::conditional<kBytes == 8, uint2, uint32_t>::type>::type;
    union {
        V v;
        T e[N];
    } u;
#pragma unroll
    for (int i = 0; i < N; ++i) u.e[i] = Elem<T>::from_float(x[i]);
    *reinterpret_cast<V *>(dst) = u.v;
}

template <typename T, int D, int R>
__global__ void __launch_bounds__(R == 1 ? 128 : R * 32) lse_reduce_kernel(const DecodeParams p) {
    constexpr int U = kReduceBatch;
    constexpr int VL = D / 32;             // floats per lane
    using V = ReduceVec<VL>;
    using VT = typename V::type;
    constexpr int NS = R == 1 ? 1 : R;     // shared-memory states (unused with R == 1)
    __shared__ float s_m[NS];
    __shared__ float s_den[NS];
    __shared__ __align__(16) float s_acc[NS][D];

    pdl_wait_primary();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // R == 1: warp-uniform row; R > 1: CTA-uniform row (so the returns below keep every
    // warp of a CTA that reaches the barrier together)
    const int row = R == 1 ? blockIdx.x * 4 + warp : blockIdx.x;
    const int wr = R == 1 ? 0 : warp;      // the warp's index within its row
    if (row >= p.S * p.Hq) return;
    const int s = row / p.Hq;
    const int L = p.context_lens[s];
    if (L < 1 || L > (p.maxB << p.bshift)) return;
    const int nblk = (L + kBlock - 1) / kBlock;
    const int np = (nblk + p.part_blocks - 1) / p.part_blocks;
    if (np <= 1) return;
    const float2 *ml = reinterpret_cast<const float2 *>(p.ws_ml) + (size_t)row * p.pmax;
    const float *ob = p.ws_o + (size_t)row * p.pmax * D + lane * VL;

    float M = -INFINITY, den = 0.f, acc[VL];
#pragma unroll
    for (int k = 0; k < VL; ++k) acc[k] = 0.f;
    for (int i0 = wr; i0 < np; i0 += R * U) {
        float2 mlv[U];
        VT v[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int i = i0 + R * u;
            if (i < np) {
                mlv[u] = ml[i];
                v[u] = *reinterpret_cast<const VT *>(ob + (size_t)i * D);
            } else {
                mlv[u] = make_float2(-INFINITY, 0.f);
            }
        }
        float bm = M;
#pragma unroll
        for (int u = 0; u < U; ++u) bm = fmaxf(bm, mlv[u].x);
        if (bm > M) {  // the batch raises the running max: rescale what is summed so far
            const float a = M == -INFINITY ? 0.f : exp2f(M - bm);
            den *= a;
#pragma unroll
            for (int k = 0; k < VL; ++k) acc[k] *= a;
            M = bm;
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            if (mlv[u].x != -INFINITY) {
                const float w = exp2f(mlv[u].x - M);
                den = fmaf(w, mlv[u].y, den);
#pragma unroll
                for (int k = 0; k < VL; ++k) acc[k] = fmaf(w, V::get(v[u], k), acc[k]);
            }
        }
    }

    if constexpr (R == 1) {
        const float inv = 1.f / den;
        float x[VL];
#pragma unroll
        for (int k = 0; k < VL; ++k) x[k] = acc[k] * inv;
        store_vec<T, VL>(static_cast<T *>(p.out) + (size_t)row * D + lane * VL, x);
    } else {
        constexpr int E = 16 / sizeof(T);  // output elements per 16-byte store
#pragma unroll
        for (int k = 0; k < VL; ++k) s_acc[warp][lane * VL + k] = acc[k];
        if (lane == 0) {
            s_m[warp] = M;
            s_den[warp] = den;
        }
        __syncthreads();
        for (int idx = threadIdx.x; idx < D / E; idx += R * 32) {
            float Mx = -INFINITY;
#pragma unroll
            for (int w = 0; w < R; ++w) Mx = fmaxf(Mx, s_m[w]);
            float a[R], dsum = 0.f;
#pragma unroll
            for (int w = 0; w < R; ++w) {
                a[w] = s_m[w] == -INFINITY ? 0.f : exp2f(s_m[w] - Mx);
                dsum = fmaf(a[w], s_den[w], dsum);
            }
            const float inv = 1.f / dsum;
            float x[E];
#pragma unroll
            for (int e = 0; e < E; ++e) {
                float t = 0.f;
#pragma unroll
                for (int w = 0; w < R; ++w) t = fmaf(a[w], s_acc[w][idx * E + e], t);
                x[e] = t * inv;
            }
            store_row<T, E>(static_cast<T *>(p.out) + (size_t)row * D + idx * E, x);
        }
    }
}

}  // namespace pkv
