// FP8 (E4M3) forward pass on sm_100a: block quantisation of Q, K, V and the
// attention forward on the quantised tiles.
//
// FlashAttention-3 page: FP8 computation through block quantisation (its
// other ingredient, incoherent processing, is not built here). Reading taken
// where the page gives no detail: one fp32 scale per block of 128 consecutive
// rows of a (batch, head) plane, s = amax / 448 (s = 1 for an all-zero block),
// code = E4M3(x / s), round to nearest even, divisions in IEEE fp32. Q and K
// get a scale per 128-row block; V gets one scale per plane (the scale then
// factors out of the P V sum) and is stored transposed, [plane, d, Np] with
// Np = 128 ceil(N / 128) and zero codes past N, so that it is a K-major MMA
// operand like Q and K.
//
// Kernels:
//   fp8_amax_kernel      largest |x| per (plane, 128-row block), into scales
//   fp8_quant_kernel     codes from x and the block (or plane) maximum,
//                        row-major or transposed
//   fp8_scales_kernel    replaces each maximum with its scale (one thread per
//                        plane, after every block has read the maxima)
//   attn_fwd_fp8_kernel  one 128-row query tile of one (batch, head) per block:
//                        S = Q8 K8^T with tcgen05.mma kind::f8f6f4 (E4M3 x E4M3,
//                        fp32 accumulator in TMEM), online softmax in fp32 with
//                        the block scales folded into the exp2 argument, P
//                        rounded to E4M3 into shared memory (128-byte swizzle),
//                        O += P8 V8 with both operands K-major in shared
//                        memory; O x s_v / l and the LSE in the epilogue.
// The attention kernel: 192 threads, warps 0-3 softmax (thread = query row =
// TMEM lane), warp 4 the MMA issuer, warp 5 the TMA producer. S is double
// buffered in TMEM, K/V tiles go through a 3-slot ring, P through two buffers.
// O is rescaled lazily: only when a row's running maximum grows by more than
// 8 (log2 units), so P stays at most 2^8, inside E4M3's range. Every wait is
// bounded.
#pragma once

#include <cuda_fp8.h>

#include "sm100_ptx.cuh"

namespace eab {

// Two floats to two E4M3 codes (round to nearest even, saturating at +-448);
// `lo` goes to the low byte.
__device__ __forceinline__ uint16_t e4m3x2(float lo, float hi) {
    return static_cast<uint16_t>(__nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE, __NV_E4M3));
}

// D(tmem) = A(smem) * B(smem) (+ D when accumulate != 0), kind::f8f6f4.
__device__ __forceinline__ void mma_f8_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// ------------------------------------------------------- quantisation ----

struct QuantParams {
    const __nv_bfloat16* x;  // [planes, N, D]
    uint8_t* codes;          // [planes, N, D], or [planes, D, Np] when transposed
    float* scales;           // [planes, nblk]: maxima after the first kernel, scales after the last
    int planes, N, nblk, Np, per_plane;
};

template <int D>
__global__ void __launch_bounds__(256) fp8_amax_kernel(const QuantParams p) {
    const int blk = blockIdx.x, plane = blockIdx.y;
    const int r0 = blk * 128, rows = min(128, p.N - r0);
    const __nv_bfloat16* src = p.x + (static_cast<size_t>(plane) * p.N + r0) * D;
    float m = 0.f;
    for (int i = threadIdx.x; i < rows * D / 8; i += 256) {
        const uint4 u = reinterpret_cast<const uint4*>(src)[i];
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(h[e]);
            m = fmaxf(m, fmaxf(fabsf(f.x), fabsf(f.y)));
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    __shared__ float wm[8];
    if ((threadIdx.x & 31) == 0) wm[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        float t = wm[0];
        for (int w = 1; w < 8; ++w) t = fmaxf(t, wm[w]);
        p.scales[static_cast<size_t>(plane) * p.nblk + blk] = t;
    }
}

__device__ __forceinline__ float fp8_scale_of(float amax) { return amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f; }

template <int D, bool TRANSPOSE>
__global__ void __launch_bounds__(256) fp8_quant_kernel(const QuantParams p) {
    const int blk = blockIdx.x, plane = blockIdx.y;
    const int r0 = blk * 128, rows = min(128, p.N - r0);
    const float* mx = p.scales + static_cast<size_t>(plane) * p.nblk;
    float m = mx[blk];
    if (p.per_plane) {
        m = 0.f;
        for (int i = 0; i < p.nblk; ++i) m = fmaxf(m, mx[i]);
    }
    const float s = fp8_scale_of(m);
    const __nv_bfloat16* src = p.x + (static_cast<size_t>(plane) * p.N + r0) * D;
    if (!TRANSPOSE) {
        uint8_t* dst = p.codes + (static_cast<size_t>(plane) * p.N + r0) * D;
        for (int i = threadIdx.x; i < rows * D / 8; i += 256) {
            const uint4 u = reinterpret_cast<const uint4*>(src)[i];
            const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
            uint16_t c[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 f = __bfloat1622float2(h[e]);
                c[e] = e4m3x2(__fdiv_rn(f.x, s), __fdiv_rn(f.y, s));
            }
            reinterpret_cast<uint2*>(dst)[i] =
                make_uint2(uint32_t(c[0]) | (uint32_t(c[1]) << 16), uint32_t(c[2]) | (uint32_t(c[3]) << 16));
        }
    } else {
        // codes of the block's 128 rows (zero past N), then written out as D rows
        // of 128 keys each
        __shared__ uint8_t tile[128][D + 16];
        for (int i = threadIdx.x; i < 128 * D / 8; i += 256) {
            const int r = i / (D / 8), c8 = (i % (D / 8)) * 8;
            uint16_t c[4] = {0, 0, 0, 0};
            if (r < rows) {
                const uint4 u = *reinterpret_cast<const uint4*>(src + static_cast<size_t>(r) * D + c8);
                const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 f = __bfloat1622float2(h[e]);
                    c[e] = e4m3x2(__fdiv_rn(f.x, s), __fdiv_rn(f.y, s));
                }
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                tile[r][c8 + 2 * e] = uint8_t(c[e] & 0xff);
                tile[r][c8 + 2 * e + 1] = uint8_t(c[e] >> 8);
            }
        }
        __syncthreads();
        uint8_t* dst = p.codes + static_cast<size_t>(plane) * D * p.Np + r0;
        for (int i = threadIdx.x; i < D * 8; i += 256) {
            const int t = i >> 3, k0 = (i & 7) * 16;  // dimension t, keys [k0, k0 + 16)
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e)
                w[e] = uint32_t(tile[k0 + 4 * e][t]) | (uint32_t(tile[k0 + 4 * e + 1][t]) << 8) |
                       (uint32_t(tile[k0 + 4 * e + 2][t]) << 16) | (uint32_t(tile[k0 + 4 * e + 3][t]) << 24);
            *reinterpret_cast<uint4*>(dst + static_cast<size_t>(t) * p.Np + k0) = make_uint4(w[0], w[1], w[2], w[3]);
        }
    }
}

__global__ void fp8_scales_kernel(const QuantParams p) {
    const int plane = blockIdx.x * blockDim.x + threadIdx.x;
    if (plane >= p.planes) return;
    float* mx = p.scales + static_cast<size_t>(plane) * p.nblk;
    float pm = 0.f;
    for (int i = 0; i < p.nblk; ++i) pm = fmaxf(pm, mx[i]);
    for (int i = 0; i < p.nblk; ++i) mx[i] = fp8_scale_of(p.per_plane ? pm : mx[i]);
}

// ------------------------------------------------------------ attention ----

struct Fp8Params {
    const float* sq;  // [B, Hq, nblk]
    const float* sk;  // [B, Hkv, nblk]
    const float* sv;  // [B, Hkv, nblk] (one value per plane)
    __nv_bfloat16* o; // [B, Hq, N, 128]
    float* lse;       // [B, Hq, N]
    int B, Hq, Hkv, N, nblk;
    float scale_log2;
};

struct Fp8Cfg {
    static constexpr int D = 128, BM = 128, BN = 128, STAGES = 3;
    static constexpr int TILE = 128 * 128;  // bytes of one 128 x 128 E4M3 tile
    static constexpr int NUM_THREADS = 192;
    // [Q][K x STAGES][V x STAGES][P x 2][barriers]
    static constexpr int SMEM_BYTES = 1024 + TILE * (1 + 2 * STAGES + 2) + 32 * 8 + 16;
};

template <bool CAUSAL>
__global__ void __launch_bounds__(192, 1)
    attn_fwd_fp8_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_vt, const Fp8Params p) {
    using C = Fp8Cfg;
    constexpr int TILE = C::TILE, STAGES = C::STAGES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = smem;
    uint8_t* sK = sQ + TILE;               // [STAGES]
    uint8_t* sV = sK + STAGES * TILE;      // [STAGES], rows = head dimension, 128 keys each
    uint8_t* sP = sV + STAGES * TILE;      // [2]
    uint64_t* bars = reinterpret_cast<uint64_t*>(sP + 2 * TILE);
    uint64_t* q_full = bars;               // Q tile loaded
    uint64_t* kv_full = bars + 1;          // [STAGES] K and V tiles of a slot loaded
    uint64_t* kv_empty = bars + 4;         // [STAGES] slot read by S and P V
    uint64_t* s_full = bars + 7;           // [2] S buffer complete
    uint64_t* s_free = bars + 9;           // [2] S buffer read into registers (4 warp arrivals)
    uint64_t* p_full = bars + 11;          // [2] P buffer written (4 warp arrivals)
    uint64_t* pv_done = bars + 13;         // [2] P V of the buffer complete
    uint64_t* fin = bars + 15;             // every MMA done
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 16);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_t = (p.N + 127) / 128;
    const int qt = CAUSAL ? n_t - 1 - static_cast<int>(blockIdx.x) : static_cast<int>(blockIdx.x);
    const int bh = blockIdx.y, b = bh / p.Hq, h = bh % p.Hq;
    const int kvp = b * p.Hkv + h / (p.Hq / p.Hkv);  // key/value plane
    const int nk = CAUSAL ? qt + 1 : n_t;

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int i = 0; i < STAGES; ++i) {
            mbar_init(&kv_full[i], 1);
            mbar_init(&kv_empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s_full[i], 1);
            mbar_init(&s_free[i], 4);
            mbar_init(&p_full[i], 4);
            mbar_init(&pv_done[i], 1);
        }
        mbar_init(fin, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 4) {
        tmem_alloc(tmem_holder, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;  // S buffers at columns 0 and 128, O at 256

    if (warp == 5) {
        // ------------------------------------------------------ producer ----
        if (lane == 0) {
            mbar_arrive_expect_tx(q_full, TILE);
            tma_load_3d(sQ, &tm_q, q_full, 0, qt * 128, bh);
            int j = 0;
            for (; j < nk; ++j) {
                const int slot = j % STAGES;
                if (j >= STAGES && !mbar_wait(&kv_empty[slot], ((j / STAGES) - 1) & 1, abort_flag)) break;
                mbar_arrive_expect_tx(&kv_full[slot], 2 * TILE);
                tma_load_3d(sK + slot * TILE, &tm_k, &kv_full[slot], 0, j * 128, kvp);
                tma_load_3d(sV + slot * TILE, &tm_vt, &kv_full[slot], j * 128, 0, kvp);
            }
            // let every copy in flight land before the CTA can exit
            mbar_wait(q_full, 0, nullptr);
            for (int i = max(0, j - STAGES); i < j; ++i) mbar_wait(&kv_full[i % STAGES], (i / STAGES) & 1, nullptr);
        }
    } else if (warp == 4) {
        // ---------------------------------------------------- MMA issuer ----
        if (lane == 0) {
            // E4M3 x E4M3 -> F32, both operands K-major: the kind::f8f6f4 format
            // code of E4M3 is 0, so the descriptor bits match make_idesc's
            constexpr uint32_t idesc = make_idesc(128, 128, 0, 0, 0);
            const uint32_t q_addr = smem_addr(sQ);
            auto issue_s = [&](int j) -> bool {
                const int slot = j % STAGES, sb = j & 1;
                if (!mbar_wait(&kv_full[slot], (j / STAGES) & 1, abort_flag)) return false;
                if (j >= 2 && !mbar_wait(&s_free[sb], ((j >> 1) - 1) & 1, abort_flag)) return false;
                tc_fence_after();
                const uint32_t k_addr = smem_addr(sK + slot * TILE);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)  // 32 bytes = 32 elements of K per MMA
                    mma_f8_ss(tmem + sb * 128, make_sdesc_sw128(q_addr + kk * 32, 16, 1024),
                              make_sdesc_sw128(k_addr + kk * 32, 16, 1024), idesc, kk > 0 ? 1u : 0u);
                tc_commit(&s_full[sb]);
                return true;
            };
            bool ok = mbar_wait(q_full, 0, abort_flag) && issue_s(0);
            for (int j = 0; ok && j < nk; ++j) {
                // S(j + 1) goes ahead of P V(j) so that it is ready when the
                // softmax finishes P(j)
                if (j + 1 < nk && !issue_s(j + 1)) {
                    ok = false;
                    break;
                }
                const int slot = j % STAGES, pb = j & 1;
                if (!mbar_wait_spin(&p_full[pb], (j >> 1) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t p_addr = smem_addr(sP + pb * TILE), v_addr = smem_addr(sV + slot * TILE);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_f8_ss(tmem + 256, make_sdesc_sw128(p_addr + kk * 32, 16, 1024),
                              make_sdesc_sw128(v_addr + kk * 32, 16, 1024), idesc, (j > 0 || kk > 0) ? 1u : 0u);
                tc_commit(&pv_done[pb]);
                tc_commit(&kv_empty[slot]);
            }
            tc_commit(fin);
            mbar_wait(fin, 0, nullptr);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------- softmax ----
        const int r = warp * 32 + lane;
        const int q_row = qt * 128 + r;
        const uint32_t lb = uint32_t(warp * 32) << 16;
        const float sq = p.sq[static_cast<size_t>(bh) * p.nblk + qt];
        const float* skp = p.sk + static_cast<size_t>(kvp) * p.nblk;
        float m_used = -INFINITY, l = 0.f;
        bool ok = true;
        for (int j = 0; j < nk; ++j) {
            const int sb = j & 1;
            if (!__all_sync(0xffffffffu, mbar_wait(&s_full[sb], (j >> 1) & 1, abort_flag))) {
                ok = false;
                break;
            }
            tc_fence_after();
            uint32_t sr0[64], sr1[64];
            tmem_ld64(tmem + lb + sb * 128, sr0);
            tmem_ld64(tmem + lb + sb * 128 + 64, sr1);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s_free[sb]);
            // scores in log2 units: S8 x s_q x s_k(j) x scale x log2(e)
            const float c = p.scale_log2 * sq * skp[j];
            const int k0 = j * 128;
            const int lim = min(p.N - k0, CAUSAL ? q_row - k0 + 1 : 128);  // visible keys: col < lim
            float x[128];
            float tmax = -INFINITY;
#pragma unroll
            for (int i = 0; i < 128; ++i) {
                x[i] = i < lim ? __uint_as_float(i < 64 ? sr0[i] : sr1[i - 64]) * c : -INFINITY;
                tmax = fmaxf(tmax, x[i]);
            }
            float factor = 1.f;
            if (j == 0) {
                m_used = tmax;
            } else if (tmax > m_used + 8.f) {
                factor = ex2_approx(m_used - tmax);
                m_used = tmax;
            }
            float rs = 0.f;
            uint32_t pk[32];
#pragma unroll
            for (int i = 0; i < 128; i += 4) {
                const float p0 = ex2_approx(x[i] - m_used), p1 = ex2_approx(x[i + 1] - m_used);
                const float p2 = ex2_approx(x[i + 2] - m_used), p3 = ex2_approx(x[i + 3] - m_used);
                rs += (p0 + p1) + (p2 + p3);
                pk[i / 4] = uint32_t(e4m3x2(p0, p1)) | (uint32_t(e4m3x2(p2, p3)) << 16);
            }
            l = l * factor + rs;
            // P buffer sb was last read by P V(j - 2); O must hold every earlier
            // P V before it is rescaled
            const bool rescale = __any_sync(0xffffffffu, factor != 1.f);
            bool w_ok = true;
            if (rescale && j >= 1)
                w_ok = mbar_wait(&pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1, abort_flag);
            else if (j >= 2)
                w_ok = mbar_wait(&pv_done[sb], ((j >> 1) - 1) & 1, abort_flag);
            if (!__all_sync(0xffffffffu, w_ok)) {
                ok = false;
                break;
            }
            if (rescale) {
                tc_fence_after();
#pragma unroll
                for (int cch = 0; cch < 4; ++cch) {
                    uint32_t ov[32];
                    tmem_ld32(tmem + lb + 256 + cch * 32, ov);
#pragma unroll
                    for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * factor);
                    tmem_st32(tmem + lb + 256 + cch * 32, ov);
                }
                tmem_st_wait();
            }
            // P row into the 128-byte-swizzled K-major tile: 16-byte chunk cc of
            // row r sits at chunk position cc ^ (r & 7)
            uint8_t* prow = sP + sb * TILE + r * 128;
#pragma unroll
            for (int cc = 0; cc < 8; ++cc)
                *reinterpret_cast<uint4*>(prow + ((cc ^ (r & 7)) << 4)) =
                    make_uint4(pk[4 * cc], pk[4 * cc + 1], pk[4 * cc + 2], pk[4 * cc + 3]);
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&p_full[sb]);
        }
        // epilogue: O x s_v / l in bf16, LSE = ln 2 (m + log2 l)
        if (ok && __all_sync(0xffffffffu, mbar_wait(fin, 0, abort_flag))) {
            tc_fence_after();
            const float f = p.sv[static_cast<size_t>(kvp) * p.nblk] / l;
            __nv_bfloat16* dst = p.o + (static_cast<size_t>(bh) * p.N + (q_row < p.N ? q_row : 0)) * 128;
#pragma unroll
            for (int cch = 0; cch < 4; ++cch) {
                uint32_t ov[32];
                tmem_ld32(tmem + lb + 256 + cch * 32, ov);
                if (q_row < p.N) {
#pragma unroll
                    for (int i = 0; i < 32; i += 8)
                        *reinterpret_cast<uint4*>(dst + cch * 32 + i) = make_uint4(
                            pack_bf16x2(__uint_as_float(ov[i]) * f, __uint_as_float(ov[i + 1]) * f),
                            pack_bf16x2(__uint_as_float(ov[i + 2]) * f, __uint_as_float(ov[i + 3]) * f),
                            pack_bf16x2(__uint_as_float(ov[i + 4]) * f, __uint_as_float(ov[i + 5]) * f),
                            pack_bf16x2(__uint_as_float(ov[i + 6]) * f, __uint_as_float(ov[i + 7]) * f));
                }
            }
            if (q_row < p.N)
                p.lse[static_cast<size_t>(bh) * p.N + q_row] = (m_used + log2f(l)) * 0.69314718055994530942f;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 4) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace eab
