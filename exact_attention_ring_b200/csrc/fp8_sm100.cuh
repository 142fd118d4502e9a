// FP8 (E4M3) forward pass on sm_100a: block quantisation of Q, K, V and the
// attention forward on the quantised tiles.
//
// FlashAttention-3 page: FP8 computation through block quantisation and
// incoherent processing (a random orthogonal rotation of Q and K that spreads
// outlier coordinates before they are quantised). Reading taken
// where the page gives no detail: one fp32 scale per block of 128 consecutive
// rows of a (batch, head) plane, s = amax / 448 (s = 1 for an all-zero block),
// code = E4M3(x / s), round to nearest even, divisions in IEEE fp32. Q and K
// get a scale per 128-row block; V gets one scale per plane (the scale then
// factors out of the P V sum) and is stored transposed, [plane, d, Np] with
// Np = 128 ceil(N / 128) and zero codes past N, so that it is a K-major MMA
// operand like Q and K.
//
// Kernels:
//   fp8_quant_rows_kernel  per-block scales and row-major codes of Q or K in
//                        one pass, optionally after the rotation
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
// TMEM lane), warp 4 the MMA issuer, warp 5 the TMA producer. The softmax reads
// S into registers at once, so one S buffer in TMEM suffices (S(j+1) is
// computed while the softmax works on tile j); K/V tiles go through a 2-slot
// ring and P through one shared-memory tile, so that two blocks share an SM (256
// TMEM columns, about 97 KB of shared memory each): one block's MMAs overlap the
// other's softmax.
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
    const float* signs;      // [D] +1 / -1: the random signs of the rotation (fp8_quant_rows_kernel<D, true>)
    float rot_scale;         // fp32 value nearest 1 / sqrt(D)
};

// One pass over one 128-row block of a plane, for the per-block, row-major codes
// of Q and K: each warp holds 16 rows in registers (lane l has elements
// l*E .. l*E+E-1, E = D/32), optionally applies the rotation of incoherent
// processing (FlashAttention-3 page, FP8 paragraph; reading: y = H (sigma o x) /
// sqrt(D), H the Sylvester Hadamard matrix, sigma random signs shared by Q and
// K), then takes the block maximum, its scale and the codes. The rotation is the
// fast Walsh-Hadamard transform in fp32 with butterflies (a, b) -> (a + b, a - b)
// of span 1, 2, ..., D/2 in that order (spans below E inside a lane, the rest
// across lanes by shuffles) and one multiplication by rot_scale: every element
// takes exactly the fp32 operations of the transform's definition, in its order.
template <int D, bool ROTATE>
__global__ void __launch_bounds__(256) fp8_quant_rows_kernel(const QuantParams p) {
    constexpr int E = D / 32, RPW = 16;
    const int blk = blockIdx.x, plane = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r0 = blk * 128, rows = min(128, p.N - r0);
    const __nv_bfloat16* src = p.x + (static_cast<size_t>(plane) * p.N + r0) * D;
    float v[RPW][E];
#pragma unroll
    for (int i = 0; i < RPW; ++i) {
        const int r = warp * RPW + i;
        if (r < rows) {
            if constexpr (E == 4) {
                const uint2 u = *reinterpret_cast<const uint2*>(src + static_cast<size_t>(r) * D + lane * E);
                const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
                const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
                v[i][0] = a.x; v[i][1] = a.y; v[i][2] = b.x; v[i][3] = b.y;
            } else {
                const uint32_t u = *reinterpret_cast<const uint32_t*>(src + static_cast<size_t>(r) * D + lane * E);
                const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u));
                v[i][0] = a.x; v[i][1] = a.y;
            }
        } else {
#pragma unroll
            for (int e = 0; e < E; ++e) v[i][e] = 0.f;
        }
    }
    if constexpr (ROTATE) {
        float sg[E];
#pragma unroll
        for (int e = 0; e < E; ++e) sg[e] = p.signs[lane * E + e];
#pragma unroll
        for (int i = 0; i < RPW; ++i) {
#pragma unroll
            for (int e = 0; e < E; ++e) v[i][e] = sg[e] * v[i][e];
#pragma unroll
            for (int h = 1; h < E; h *= 2)
#pragma unroll
                for (int b = 0; b < E; b += 2 * h)
#pragma unroll
                    for (int t = b; t < b + h; ++t) {
                        const float a = v[i][t], c = v[i][t + h];
                        v[i][t] = __fadd_rn(a, c);
                        v[i][t + h] = __fsub_rn(a, c);
                    }
#pragma unroll
            for (int h = E; h < D; h *= 2) {
                const int m = h / E;  // partner lane of element lane*E + e is lane ^ m
                const bool lower = (lane & m) == 0;
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    const float u = __shfl_xor_sync(0xffffffffu, v[i][e], m);
                    v[i][e] = lower ? __fadd_rn(v[i][e], u) : __fsub_rn(u, v[i][e]);
                }
            }
#pragma unroll
            for (int e = 0; e < E; ++e) v[i][e] = __fmul_rn(v[i][e], p.rot_scale);
        }
    }
    float m = 0.f;
#pragma unroll
    for (int i = 0; i < RPW; ++i)
#pragma unroll
        for (int e = 0; e < E; ++e) m = fmaxf(m, fabsf(v[i][e]));  // rows past N hold zeros
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    __shared__ float wm[8];
    if (lane == 0) wm[warp] = m;
    __syncthreads();
    float amax = wm[0];
#pragma unroll
    for (int w = 1; w < 8; ++w) amax = fmaxf(amax, wm[w]);
    const float sc = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
    if (threadIdx.x == 0) p.scales[static_cast<size_t>(plane) * p.nblk + blk] = sc;
    uint8_t* dst = p.codes + (static_cast<size_t>(plane) * p.N + r0) * D;
#pragma unroll
    for (int i = 0; i < RPW; ++i) {
        const int r = warp * RPW + i;
        if (r >= rows) break;
        if constexpr (E == 4) {
            const uint32_t c = uint32_t(e4m3x2(__fdiv_rn(v[i][0], sc), __fdiv_rn(v[i][1], sc))) |
                               (uint32_t(e4m3x2(__fdiv_rn(v[i][2], sc), __fdiv_rn(v[i][3], sc))) << 16);
            *reinterpret_cast<uint32_t*>(dst + static_cast<size_t>(r) * D + lane * E) = c;
        } else {
            *reinterpret_cast<uint16_t*>(dst + static_cast<size_t>(r) * D + lane * E) =
                e4m3x2(__fdiv_rn(v[i][0], sc), __fdiv_rn(v[i][1], sc));
        }
    }
}

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
    static constexpr int D = 128, BM = 128, BN = 128, STAGES = 2;
    static constexpr int TILE = 128 * 128;  // bytes of one 128 x 128 E4M3 tile
    static constexpr int NUM_THREADS = 192;
    static constexpr uint32_t TMEM_COLS = 256;  // S [0, 128), O [128, 256)
    // [Q][K x STAGES][V x STAGES][P][barriers]: two blocks fit one SM (shared
    // memory and TMEM), so one block's MMAs overlap the other's softmax
    static constexpr int SMEM_BYTES = 1024 + TILE * (1 + 2 * STAGES + 1) + 16 * 8 + 16;
};

template <bool CAUSAL>
__global__ void __launch_bounds__(192, 2)
    attn_fwd_fp8_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_vt, const Fp8Params p) {
    using C = Fp8Cfg;
    constexpr int TILE = C::TILE, STAGES = C::STAGES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = smem;
    uint8_t* sK = sQ + TILE;               // [STAGES]
    uint8_t* sV = sK + STAGES * TILE;      // [STAGES], rows = head dimension, 128 keys each
    uint8_t* sP = sV + STAGES * TILE;      // P (E4M3), 128 rows of 128 keys
    uint64_t* bars = reinterpret_cast<uint64_t*>(sP + TILE);
    uint64_t* q_full = bars;               // Q tile loaded
    uint64_t* kv_full = bars + 1;          // [STAGES] K and V tiles of a slot loaded
    uint64_t* kv_empty = bars + 3;         // [STAGES] slot read by S and P V
    uint64_t* s_full = bars + 5;           // S complete
    uint64_t* s_free = bars + 6;           // S read into registers (4 warp arrivals)
    uint64_t* p_full = bars + 7;           // P written (4 warp arrivals)
    uint64_t* pv_done = bars + 8;          // P V complete
    uint64_t* fin = bars + 9;              // every MMA done
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 10);
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
        mbar_init(s_full, 1);
        mbar_init(s_free, 4);
        mbar_init(p_full, 4);
        mbar_init(pv_done, 1);
        mbar_init(fin, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 4) {
        tmem_alloc(tmem_holder, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

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
                const int slot = j % STAGES;
                if (!mbar_wait(&kv_full[slot], (j / STAGES) & 1, abort_flag)) return false;
                // the softmax has read S(j - 1) into registers
                if (j >= 1 && !mbar_wait(s_free, (j - 1) & 1, abort_flag)) return false;
                tc_fence_after();
                const uint32_t k_addr = smem_addr(sK + slot * TILE);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)  // 32 bytes = 32 elements of K per MMA
                    mma_f8_ss(tmem, make_sdesc_sw128(q_addr + kk * 32, 16, 1024),
                              make_sdesc_sw128(k_addr + kk * 32, 16, 1024), idesc, kk > 0 ? 1u : 0u);
                tc_commit(s_full);
                return true;
            };
            bool ok = mbar_wait(q_full, 0, abort_flag) && issue_s(0);
            for (int j = 0; ok && j < nk; ++j) {
                // S(j + 1) goes ahead of P V(j): it runs while the softmax works on P(j)
                if (j + 1 < nk && !issue_s(j + 1)) {
                    ok = false;
                    break;
                }
                const int slot = j % STAGES;
                if (!mbar_wait_spin(p_full, j & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t p_addr = smem_addr(sP), v_addr = smem_addr(sV + slot * TILE);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_f8_ss(tmem + 128, make_sdesc_sw128(p_addr + kk * 32, 16, 1024),
                              make_sdesc_sw128(v_addr + kk * 32, 16, 1024), idesc, (j > 0 || kk > 0) ? 1u : 0u);
                tc_commit(pv_done);
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
            if (!__all_sync(0xffffffffu, mbar_wait(s_full, j & 1, abort_flag))) {
                ok = false;
                break;
            }
            tc_fence_after();
            uint32_t sr[128];
            tmem_ld64(tmem + lb, reinterpret_cast<uint32_t(&)[64]>(sr[0]));
            tmem_ld64(tmem + lb + 64, reinterpret_cast<uint32_t(&)[64]>(sr[64]));
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(s_free);  // S(j + 1) may overwrite S now
            // scores in log2 units: S8 x s_q x s_k(j) x scale x log2(e), c > 0
            const float c = p.scale_log2 * sq * skp[j];
            const int k0 = j * 128;
            const int lim = min(p.N - k0, CAUSAL ? q_row - k0 + 1 : 128);  // visible keys: col < lim
            if (__any_sync(0xffffffffu, lim < 128)) {
#pragma unroll
                for (int i = 0; i < 128; ++i)
                    if (i >= lim) sr[i] = 0xff800000u;  // -inf: exp2 gives 0
            }
            float mx = -INFINITY;
#pragma unroll
            for (int i = 0; i < 128; i += 2) mx = max3(mx, __uint_as_float(sr[i]), __uint_as_float(sr[i + 1]));
            const float tmax = mx * c;
            float factor = 1.f;
            if (j == 0) {
                m_used = tmax;
            } else if (tmax > m_used + 8.f) {
                factor = ex2_approx(m_used - tmax);
                m_used = tmax;
            }
            const float2 cc2 = make_float2(c, c), negm2 = make_float2(-m_used, -m_used);
            float2 rsum[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) rsum[k] = make_float2(0.f, 0.f);
            uint32_t pk[32];
#pragma unroll
            for (int i = 0; i < 128; i += 4) {
                const float2 y0 = ffma2(make_float2(__uint_as_float(sr[i]), __uint_as_float(sr[i + 1])), cc2, negm2);
                const float2 y1 = ffma2(make_float2(__uint_as_float(sr[i + 2]), __uint_as_float(sr[i + 3])), cc2, negm2);
                const float2 p0 = make_float2(ex2_approx(y0.x), ex2_approx(y0.y));
                const float2 p1 = make_float2(ex2_approx(y1.x), ex2_approx(y1.y));
                rsum[(i >> 2) & 3] = fadd2(rsum[(i >> 2) & 3], fadd2(p0, p1));
                pk[i / 4] = uint32_t(e4m3x2(p0.x, p0.y)) | (uint32_t(e4m3x2(p1.x, p1.y)) << 16);
            }
            const float2 rs = fadd2(fadd2(rsum[0], rsum[1]), fadd2(rsum[2], rsum[3]));
            l = l * factor + (rs.x + rs.y);
            // P V(j - 1) must be complete: it still reads the P buffer, and O must
            // hold it before a rescale
            if (j >= 1 && !__all_sync(0xffffffffu, mbar_wait(pv_done, (j - 1) & 1, abort_flag))) {
                ok = false;
                break;
            }
            if (__any_sync(0xffffffffu, factor != 1.f)) {
                tc_fence_after();
#pragma unroll
                for (int cch = 0; cch < 4; ++cch) {
                    uint32_t ov[32];
                    tmem_ld32(tmem + lb + 128 + cch * 32, ov);
#pragma unroll
                    for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * factor);
                    tmem_st32(tmem + lb + 128 + cch * 32, ov);
                }
                tmem_st_wait();
            }
            // P row into the 128-byte-swizzled K-major tile: 16-byte chunk cc of
            // row r sits at chunk position cc ^ (r & 7)
            uint8_t* prow = sP + r * 128;
#pragma unroll
            for (int cc = 0; cc < 8; ++cc)
                *reinterpret_cast<uint4*>(prow + ((cc ^ (r & 7)) << 4)) =
                    make_uint4(pk[4 * cc], pk[4 * cc + 1], pk[4 * cc + 2], pk[4 * cc + 3]);
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(p_full);
        }
        // epilogue: O x s_v / l in bf16, LSE = ln 2 (m + log2 l)
        if (ok && __all_sync(0xffffffffu, mbar_wait(fin, 0, abort_flag))) {
            tc_fence_after();
            const float f = p.sv[static_cast<size_t>(kvp) * p.nblk] / l;
            __nv_bfloat16* dst = p.o + (static_cast<size_t>(bh) * p.N + (q_row < p.N ? q_row : 0)) * 128;
#pragma unroll
            for (int cch = 0; cch < 4; ++cch) {
                uint32_t ov[32];
                tmem_ld32(tmem + lb + 128 + cch * 32, ov);
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
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

}  // namespace eab
