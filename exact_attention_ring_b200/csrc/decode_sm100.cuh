// Split-KV single-query decode and the log-sum-exp weighted combine.
//
// Flash-Decoding (FlashAttention V2 page): for one query token the key/value
// range is split across thread blocks so that long caches still fill the GPU;
// each split produces a normalised partial output and its log-sum-exp, and a
// second kernel merges them (FlashAttention-3 page, split-K combine).
//
// Decode is bound by reading K and V from HBM once (about 4 FLOP per byte), so
// it runs on the CUDA cores, not the tensor cores. B200 mapping, 256 threads
// (two warps per SM sub-partition, so every thread may hold up to 255 registers):
//   warps 6, 7  TMA producers: 96-key K and V tiles of this split into a ring
//               of shared-memory stages (128-byte swizzle, zero fill past L).
//               One issuing thread streams TMA boxes one after another, so the
//               boxes of every stage are split between two threads, and boxes
//               are large (96 rows, 12 KB) because each box costs about the same
//               time whatever its size.
//   warps 0-5   each owns 16 keys of every stage, 8 at a time. Lane =
//               quarter*8 + key: the lane dots its quarter of the key row with
//               the GH query heads held in registers (the swizzle makes the 8
//               keys of a quarter-warp hit distinct banks), the quarters are
//               summed with two shuffles, the warp keeps its own online-softmax
//               state (log2 units, exp2), and for O += p v each lane owns D/32
//               output columns of every head. Products use packed f32x2 FMAs.
//   end         the six warps' states are merged in shared memory into the
//               split's partial (O_s / l_s, lse_s).
#pragma once

#include "sm100_ptx.cuh"

namespace eab {

struct DecodeParams {
    const __nv_bfloat16* q;  // [B, Hq, D]
    float* o_part;           // [B, Hq, S, D]
    float* lse_part;         // [B, Hq, S]
    int B, Hq, Hkv, L, S, chunk, groups;  // groups = (Hq/Hkv) / GH; chunk a multiple of TK
    float scale_log2;
};

template <int D, int GH>
struct DecCfg {
    static constexpr int TK = 96;       // keys per stage
    static constexpr int STAGES = (D == 128) ? 4 : 8;
    static constexpr int WARPS = 6;     // compute warps
    static constexpr int KPW = TK / WARPS;  // keys per warp per stage (two groups of 8)
    static constexpr int CHUNKS = D / 64;
    static constexpr int BOX_BYTES = TK * 128;
    static constexpr int TILE_BYTES = TK * D * 2;
    static constexpr int STAGE_BYTES = 2 * TILE_BYTES;  // K tile then V tile
    static constexpr int BOXES = 2 * CHUNKS;            // boxes per stage
    static constexpr int QPL = D / 4;   // query elements per lane (one quarter of the row)
    static constexpr int CPL = D / 32;  // output columns per lane
    static constexpr int NUM_THREADS = 32 * WARPS + 64;
    // ring | p[WARPS][8 keys][GH] | m,l [WARPS][GH] | o [WARPS][GH][D] | barriers
    static constexpr int P_OFF = STAGES * STAGE_BYTES;
    static constexpr int ML_OFF = P_OFF + WARPS * 8 * GH * 4;
    static constexpr int O_OFF = ML_OFF + 2 * WARPS * GH * 4;
    static constexpr int BAR_OFF = O_OFF + WARPS * GH * D * 4;
    static constexpr int SMEM_BYTES = 1024 + BAR_OFF + 2 * STAGES * 8 + 16;
};

// bf16 pair (one 32-bit word) -> two floats, exact.
__device__ __forceinline__ float bf_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf_hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }
__device__ __forceinline__ float2 bf_pair(uint32_t u) { return make_float2(bf_lo(u), bf_hi(u)); }

template <int D, int GH>
__global__ void __launch_bounds__(DecCfg<D, GH>::NUM_THREADS, 1)
    decode_splitkv_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                          const DecodeParams p) {
    using C = DecCfg<D, GH>;
    constexpr int TK = C::TK, STAGES = C::STAGES, WARPS = C::WARPS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float* p_s = reinterpret_cast<float*>(smem + C::P_OFF);
    float* m_s = reinterpret_cast<float*>(smem + C::ML_OFF);
    float* l_s = m_s + WARPS * GH;
    float* o_s = reinterpret_cast<float*>(smem + C::O_OFF);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
    uint64_t* empty = full + STAGES;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + STAGES);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int split = blockIdx.x;
    const int hk = blockIdx.y / p.groups, grp = blockIdx.y % p.groups;
    const int b = blockIdx.z;
    const int G = p.Hq / p.Hkv;
    const int h0 = hk * G + grp * GH;  // first query head of this block
    const int k0 = split * p.chunk;
    const int k1 = min(p.L, k0 + p.chunk);
    const int ntiles = k1 > k0 ? (k1 - k0 + TK - 1) / TK : 0;

    if (threadIdx.x == 0) {
        for (int i = 0; i < STAGES; ++i) {
            mbar_init(&full[i], C::BOXES);  // one expect_tx arrival per box
            mbar_init(&empty[i], WARPS);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();

    if (warp >= WARPS) {
        // ------------------------------------------------------ producers ---
        // box x of a stage (x < CHUNKS: K chunk x, else V chunk x - CHUNKS) is
        // issued by producer x % 2
        const int me = warp - WARPS;
        if (lane == 0 && ntiles > 0) {
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            const int z = b * p.Hkv + hk;
            int issued = 0;
            for (int t = 0; t < ntiles; ++t) {
                const int slot = t % STAGES, use = t / STAGES;
                if (use > 0 && !mbar_wait(&empty[slot], (use - 1) & 1, abort_flag)) break;
                uint8_t* dst = smem + slot * C::STAGE_BYTES;
#pragma unroll
                for (int x = 0; x < C::BOXES; ++x) {
                    if (x % 2 != me) continue;
                    const int c = x % C::CHUNKS;
                    const bool is_v = x >= C::CHUNKS;
                    mbar_arrive_expect_tx(&full[slot], C::BOX_BYTES);
                    tma_load_3d(dst + (is_v ? C::TILE_BYTES : 0) + c * C::BOX_BYTES, is_v ? &tm_v : &tm_k,
                                &full[slot], c * 64, k0 + t * TK, z);
                }
                issued = t + 1;
            }
            for (int t = max(0, issued - STAGES); t < issued; ++t)
                mbar_wait(&full[t % STAGES], (t / STAGES) & 1, nullptr);
        }
        return;  // producers take no part in the merge below (named barrier 1 counts the compute warps)
    }

    // -------------------------------------------------------- compute -------
    const int qtr = lane >> 3;  // quarter of the key row this lane dots
    const int kk = lane & 7;    // key of the current group of 8 this lane owns
    float2 qreg[GH][C::QPL / 2];
#pragma unroll
    for (int g = 0; g < GH; ++g) {
        const __nv_bfloat16* qrow = p.q + (static_cast<size_t>(b) * p.Hq + h0 + g) * D + qtr * C::QPL;
#pragma unroll
        for (int i = 0; i < C::QPL; i += 8) {
            const uint4 u = *reinterpret_cast<const uint4*>(qrow + i);
            qreg[g][i / 2 + 0] = bf_pair(u.x);
            qreg[g][i / 2 + 1] = bf_pair(u.y);
            qreg[g][i / 2 + 2] = bf_pair(u.z);
            qreg[g][i / 2 + 3] = bf_pair(u.w);
        }
    }
    float m[GH], lsum[GH];
    float2 acc[GH][C::CPL / 2];
#pragma unroll
    for (int g = 0; g < GH; ++g) {
        m[g] = -INFINITY;
        lsum[g] = 0.f;
#pragma unroll
        for (int e = 0; e < C::CPL / 2; ++e) acc[g][e] = make_float2(0.f, 0.f);
    }
    float* pw = p_s + warp * 8 * GH;

    for (int t = 0; t < ntiles; ++t) {
        const int slot = t % STAGES;
        const bool w = mbar_wait(&full[slot], (t / STAGES) & 1, abort_flag);
        if (!__all_sync(0xffffffffu, w)) break;
        const uint8_t* sK = smem + slot * C::STAGE_BYTES;
        const uint8_t* sV = sK + C::TILE_BYTES;
#pragma unroll
        for (int sub = 0; sub < C::KPW / 8; ++sub) {
            const int r = warp * C::KPW + sub * 8 + kk;  // row of this lane's key inside the stage
            // scores: this lane's quarter of key r against the GH query heads
            float2 part[GH];
#pragma unroll
            for (int g = 0; g < GH; ++g) part[g] = make_float2(0.f, 0.f);
#pragma unroll
            for (int i = 0; i < C::QPL / 8; ++i) {
                const int cc = qtr * (C::QPL / 8) + i;  // logical 16-byte chunk in the row
                const uint4 u = *reinterpret_cast<const uint4*>(sK + (cc >> 3) * C::BOX_BYTES + r * 128 +
                                                                (((cc & 7) ^ (r & 7)) << 4));
                const float2 kf[4] = {bf_pair(u.x), bf_pair(u.y), bf_pair(u.z), bf_pair(u.w)};
#pragma unroll
                for (int g = 0; g < GH; ++g)
#pragma unroll
                    for (int e = 0; e < 4; ++e) part[g] = ffma2(qreg[g][i * 4 + e], kf[e], part[g]);
            }
            const bool valid = k0 + t * TK + r < k1;
            float pr[GH];
#pragma unroll
            for (int g = 0; g < GH; ++g) {
                float sdot = part[g].x + part[g].y;
                sdot += __shfl_xor_sync(0xffffffffu, sdot, 8);
                sdot += __shfl_xor_sync(0xffffffffu, sdot, 16);
                const float s2 = valid ? sdot * p.scale_log2 : -INFINITY;
                float tmax = s2;
                tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 1));
                tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 2));
                tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 4));
                const float m_new = fmaxf(m[g], tmax);
                const float factor = (m_new == m[g]) ? 1.f : ex2_approx(m[g] - m_new);
                m[g] = m_new;
                lsum[g] *= factor;
                if (factor != 1.f) {
#pragma unroll
                    for (int e = 0; e < C::CPL / 2; ++e) {
                        acc[g][e].x *= factor;
                        acc[g][e].y *= factor;
                    }
                }
                const float m_safe = (m_new == -INFINITY) ? 0.f : m_new;
                pr[g] = ex2_approx(s2 - m_safe);
                if (qtr == 0) lsum[g] += pr[g];
            }
            if (qtr == 0) {
#pragma unroll
                for (int g = 0; g < GH; ++g) pw[kk * GH + g] = pr[g];
            }
            __syncwarp();
            // O += p v over the group's 8 keys; lane owns columns [lane*CPL, lane*CPL+CPL)
#pragma unroll
            for (int k2 = 0; k2 < 8; ++k2) {
                const int r2 = warp * C::KPW + sub * 8 + k2;
                const int byte = lane * C::CPL * 2;  // byte offset of this lane's columns in the row
                const int cc = byte >> 4;
                const uint8_t* src =
                    sV + (cc >> 3) * C::BOX_BYTES + r2 * 128 + ((((cc & 7) ^ (r2 & 7)) << 4) | (byte & 15));
                float2 vf[C::CPL / 2];
                if constexpr (C::CPL == 4) {
                    const uint2 u = *reinterpret_cast<const uint2*>(src);
                    vf[0] = bf_pair(u.x);
                    vf[1] = bf_pair(u.y);
                } else {
                    vf[0] = bf_pair(*reinterpret_cast<const uint32_t*>(src));
                }
#pragma unroll
                for (int g = 0; g < GH; ++g) {
                    const float pg = pw[k2 * GH + g];
                    const float2 pp = make_float2(pg, pg);
#pragma unroll
                    for (int e = 0; e < C::CPL / 2; ++e) acc[g][e] = ffma2(pp, vf[e], acc[g][e]);
                }
            }
            __syncwarp();
        }
        if (lane == 0) mbar_arrive(&empty[slot]);
    }

    // --------------------------------------------- merge the six warps ------
#pragma unroll
    for (int g = 0; g < GH; ++g) {
        float ls = lsum[g];
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) ls += __shfl_xor_sync(0xffffffffu, ls, off);
        if (lane == 0) {
            m_s[warp * GH + g] = m[g];
            l_s[warp * GH + g] = ls;
        }
    }
    named_barrier(1, 32 * WARPS);
#pragma unroll
    for (int g = 0; g < GH; ++g) {
        float M = m_s[g];
#pragma unroll
        for (int w2 = 1; w2 < WARPS; ++w2) M = fmaxf(M, m_s[w2 * GH + g]);
        const float f = (m[g] == -INFINITY) ? 0.f : ex2_approx(m[g] - M);
#pragma unroll
        for (int e = 0; e < C::CPL / 2; ++e) {
            o_s[(warp * GH + g) * D + lane * C::CPL + 2 * e] = acc[g][e].x * f;
            o_s[(warp * GH + g) * D + lane * C::CPL + 2 * e + 1] = acc[g][e].y * f;
        }
    }
    named_barrier(1, 32 * WARPS);
    const int tid = threadIdx.x;
    for (int idx = tid; idx < GH * D; idx += 32 * WARPS) {
        const int g = idx / D, col = idx % D;
        float M = m_s[g];
#pragma unroll
        for (int w2 = 1; w2 < WARPS; ++w2) M = fmaxf(M, m_s[w2 * GH + g]);
        float Ltot = 0.f, o = 0.f;
#pragma unroll
        for (int w2 = 0; w2 < WARPS; ++w2) {
            const float mw = m_s[w2 * GH + g];
            Ltot += (mw == -INFINITY) ? 0.f : l_s[w2 * GH + g] * ex2_approx(mw - M);
            o += o_s[(w2 * GH + g) * D + col];
        }
        const size_t u = (static_cast<size_t>(b) * p.Hq + h0 + g) * p.S + split;
        const bool empty_split = (Ltot == 0.f);
        p.o_part[u * D + col] = empty_split ? 0.f : o / Ltot;
        if (col == 0) p.lse_part[u] = empty_split ? -INFINITY : (M + log2f(Ltot)) * 0.69314718055994530942f;
    }
}

// ------------------------------------------------------------- combine ------
// One block per (b, h), D threads: M = max_s lse_s, w_s = exp(lse_s - M),
// O = sum_s w_s O_s / sum_s w_s, LSE = M + ln(sum_s w_s).
template <int D>
__global__ void __launch_bounds__(D)
    combine_kernel(const float* __restrict__ o_part, const float* __restrict__ lse_part,
                   __nv_bfloat16* __restrict__ o, float* __restrict__ lse, int S) {
    extern __shared__ float w_s[];  // S weights
    __shared__ float red[D / 32];
    __shared__ float bcast;
    const int bh = blockIdx.x, t = threadIdx.x;
    const float* lp = lse_part + static_cast<size_t>(bh) * S;

    float M = -INFINITY;
    for (int s = t; s < S; s += D) M = fmaxf(M, lp[s]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    if ((t & 31) == 0) red[t >> 5] = M;
    __syncthreads();
    if (t == 0) {
        float mm = red[0];
        for (int i = 1; i < D / 32; ++i) mm = fmaxf(mm, red[i]);
        bcast = mm;
    }
    __syncthreads();
    M = bcast;
    __syncthreads();

    float ws = 0.f;
    for (int s = t; s < S; s += D) {
        const float w = (lp[s] == -INFINITY) ? 0.f : expf(lp[s] - M);
        w_s[s] = w;
        ws += w;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ws += __shfl_xor_sync(0xffffffffu, ws, off);
    if ((t & 31) == 0) red[t >> 5] = ws;
    __syncthreads();
    if (t == 0) {
        float tot = 0.f;
        for (int i = 0; i < D / 32; ++i) tot += red[i];
        bcast = tot;
    }
    __syncthreads();
    const float wsum = bcast;

    const float* op = o_part + static_cast<size_t>(bh) * S * D + t;
    float acc = 0.f;
    for (int s = 0; s < S; ++s) acc = fmaf(w_s[s], op[static_cast<size_t>(s) * D], acc);
    const bool none = !(wsum > 0.f);
    o[static_cast<size_t>(bh) * D + t] = __float2bfloat16_rn(none ? 0.f : acc / wsum);
    if (t == 0) lse[bh] = none ? -INFINITY : M + logf(wsum);
}

}  // namespace eab
