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
//   attn_fwd_fp8_kernel  the persistent two-tile forward of attn_fwd_kernel on
//                        E4M3 tiles: S = Q8 K8^T with tcgen05.mma kind::f8f6f4
//                        (E4M3 x E4M3, fp32 accumulator in TMEM), online softmax
//                        in fp32 with the block scales folded into the exp2
//                        argument, P rounded to E4M3 into shared memory (128-byte
//                        swizzle), O += P8 V8 with both operands K-major in shared
//                        memory; O x s_v / l and the LSE in the epilogue.
// O is rescaled lazily: only when a row's running maximum grows by more than 8
// (log2 units), so P stays at most 2^8, inside E4M3's range. Every wait is
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
// of Q and K (512 threads, so that an SM holds enough blocks' loads in flight):
// each of the 16 warps holds 8 rows in registers (lane l has elements
// l*E .. l*E+E-1, E = D/32), optionally applies the rotation of incoherent
// processing (FlashAttention-3 page, FP8 paragraph; reading: y = H (sigma o x) /
// sqrt(D), H the Sylvester Hadamard matrix, sigma random signs shared by Q and
// K), then takes the block maximum, its scale and the codes. The rotation is the
// fast Walsh-Hadamard transform in fp32 with butterflies (a, b) -> (a + b, a - b)
// of span 1, 2, ..., D/2 in that order (spans below E inside a lane, the rest
// across lanes by shuffles) and one multiplication by rot_scale: every element
// takes exactly the fp32 operations of the transform's definition, in its order.
constexpr int kQuantRowsThreads = 512;
template <int D, bool ROTATE>
__global__ void __launch_bounds__(kQuantRowsThreads) fp8_quant_rows_kernel(const QuantParams p) {
    grid_dep_wait();  // the previous kernel's writes are visible from here on
    grid_dep_launch();
    constexpr int NW = kQuantRowsThreads / 32, E = D / 32, RPW = 128 / NW;
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
    __shared__ float wm[NW];
    if (lane == 0) wm[warp] = m;
    __syncthreads();
    float amax = wm[0];
#pragma unroll
    for (int w = 1; w < NW; ++w) amax = fmaxf(amax, wm[w]);
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
    grid_dep_wait();  // the previous kernel's writes are visible from here on
    grid_dep_launch();
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
    grid_dep_wait();  // the previous kernel's writes are visible from here on
    grid_dep_launch();
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
        // codes of the block's 128 rows (zero past N), transposed through shared
        // memory and written out as D rows of 128 keys each. Lane l converts keys
        // 4l .. 4l + 3 at 8 dimensions and stores, per dimension, the four codes
        // as one word (key-consecutive words: no bank conflicts); the rows of the
        // tile are 33 words apart, so the read-back of 16 keys of a dimension per
        // thread is conflict-free as well.
        __shared__ uint32_t tileT[D][33];
        const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
        const int kq = lane;  // keys 4kq .. 4kq + 3
        for (int g = warp; g < D / 8; g += 8) {
            const int c8 = g * 8;
            uint16_t c[4][4];  // [key][dimension pair]
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int r = 4 * kq + j;
#pragma unroll
                for (int e = 0; e < 4; ++e) c[j][e] = 0;
                if (r < rows) {
                    const uint4 u = *reinterpret_cast<const uint4*>(src + static_cast<size_t>(r) * D + c8);
                    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 f = __bfloat1622float2(h[e]);
                        c[j][e] = e4m3x2(__fdiv_rn(f.x, s), __fdiv_rn(f.y, s));
                    }
                }
            }
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int sh = (e & 1) * 8;
                tileT[c8 + e][kq] = uint32_t((c[0][e >> 1] >> sh) & 0xff) | (uint32_t((c[1][e >> 1] >> sh) & 0xff) << 8) |
                                    (uint32_t((c[2][e >> 1] >> sh) & 0xff) << 16) |
                                    (uint32_t((c[3][e >> 1] >> sh) & 0xff) << 24);
            }
        }
        __syncthreads();
        uint8_t* dst = p.codes + static_cast<size_t>(plane) * D * p.Np + r0;
        for (int i = threadIdx.x; i < D * 8; i += 256) {
            const int t = i >> 3, q = i & 7;  // dimension t, keys [16q, 16q + 16)
            *reinterpret_cast<uint4*>(dst + static_cast<size_t>(t) * p.Np + 16 * q) =
                make_uint4(tileT[t][4 * q], tileT[t][4 * q + 1], tileT[t][4 * q + 2], tileT[t][4 * q + 3]);
        }
    }
}

__global__ void fp8_scales_kernel(const QuantParams p) {
    grid_dep_wait();  // the previous kernel's writes are visible from here on
    grid_dep_launch();
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
    int n_qblocks;    // ceil(N / 256)
    int n_items;      // n_qblocks * B * Hq
    float scale_log2;
};

struct Fp8Cfg {
    static constexpr int D = 128, BM = 128, BN = 128, TILES = 2;
    static constexpr int TILE = 128 * 128;  // bytes of one 128 x 128 E4M3 tile
    static constexpr int SLOTS = 8;          // K and V^T tiles in load order K_0 V_0 K_1 V_1 ...
    static constexpr int STAGE_O_BYTES = 32 * 64 * 2;  // per softmax warp: 32 rows x 64 bf16
    static constexpr int NUM_THREADS = 384;
    // q_full, q_empty (2 each), slot_full, slot_empty (SLOTS each), s_full, s_free,
    // p_full, pv_done, o_free, turn, drain (2 each)
    static constexpr int NUM_BARRIERS = 4 + 2 * SLOTS + 7 * 2;
    // [Q x 2][K/V ring][P x 2][O staging][barriers]
    static constexpr int SMEM_BYTES =
        1024 + TILES * TILE + SLOTS * TILE + TILES * TILE + 8 * STAGE_O_BYTES + NUM_BARRIERS * 8 + 16;
    static constexpr uint32_t TMEM_COLS = 512;  // tile t: S [256t, 256t+128), O [256t+128, 256t+256)
};

// One work item: a 256-row query block of one (batch, head), as for attn_fwd,
// or half of one. Tile 0 holds query rows [128 q0, 128 q0 + 128), tile 1 the
// next 128 when nk1 > 0; nkv K/V tile pairs are loaded for the item.
struct Fp8Item {
    int bh, b, h, hk, q0, nk0, nk1, nkv;
};

// Of every 8 pairs of scores in a row of a tile with no masked key, this many
// take exp2 from the FMA-pipe polynomial and the rest from the MUFU (one
// warp-wide ex2 per 8 cycles per sub-partition). Measured: 2 gives 1-4 %
// over 0; 3 and more lose again to the extra issue slots. Masked tiles keep
// the MUFU throughout, whose exp2(-inf) is an exact 0.
constexpr int kFp8PolyPairs = 2;

// Largest of the 128 scores of a row (raw accumulator bits): eight independent
// chains of three-way maxima, so the pass is not one 64-deep dependency chain.
__device__ __forceinline__ float fp8_row_max(const uint32_t (&sr)[128]) {
    float m[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) m[k] = __uint_as_float(sr[k]);
#pragma unroll
    for (int i = 8; i < 120; i += 16) {
#pragma unroll
        for (int k = 0; k < 8; ++k) m[k] = max3(m[k], __uint_as_float(sr[i + k]), __uint_as_float(sr[i + 8 + k]));
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) m[k] = fmaxf(m[k], __uint_as_float(sr[120 + k]));
    return max3(max3(m[0], m[1], m[2]), max3(m[3], m[4], m[5]), fmaxf(m[6], m[7]));
}

// One row of P for a key tile: p = 2^(s c - m) for the 128 scores s of the row
// (raw accumulator bits), packed to E4M3 pairs in pk and summed into rsum.
template <int POLY>
__device__ __forceinline__ void fp8_exp_row(const uint32_t (&sr)[128], float2 cc2, float2 negm2, float2 (&rsum)[4],
                                            uint32_t (&pk)[32]) {
#pragma unroll
    for (int i = 0; i < 128; i += 4) {
        const float2 y0 = ffma2(make_float2(__uint_as_float(sr[i]), __uint_as_float(sr[i + 1])), cc2, negm2);
        const float2 y1 = ffma2(make_float2(__uint_as_float(sr[i + 2]), __uint_as_float(sr[i + 3])), cc2, negm2);
        const float2 p0 = ((i / 2) % 8 < POLY) ? exp2_poly3x2(y0) : make_float2(ex2_approx(y0.x), ex2_approx(y0.y));
        const float2 p1 = ((i / 2 + 1) % 8 < POLY) ? exp2_poly3x2(y1) : make_float2(ex2_approx(y1.x), ex2_approx(y1.y));
        rsum[(i >> 2) & 3] = fadd2(rsum[(i >> 2) & 3], fadd2(p0, p1));
        pk[i / 4] = uint32_t(e4m3x2(p0.x, p0.y)) | (uint32_t(e4m3x2(p1.x, p1.y)) << 16);
    }
}

// Item r of this CTA, false once it has none. Rounds of gridDim.x items,
// forwards in even rounds and backwards in odd ones. Without the causal mask
// every item costs the same, so a last round that would leave more than half
// the CTAs idle is dealt as 128-row halves instead (tile 0 alone), which
// shortens it to roughly the time of one tile.
template <bool CAUSAL>
__device__ __forceinline__ bool fp8_item(const Fp8Params& p, int r, Fp8Item& it) {
    const int G = gridDim.x, c = blockIdx.x;
    const int full_rounds = p.n_items / G, rem = p.n_items - full_rounds * G;
    int w, half = -1;
    if (!CAUSAL && r == full_rounds && rem > 0 && 2 * rem <= G) {
        if (c >= 2 * rem) return false;
        w = full_rounds * G + (c >> 1);
        half = c & 1;
    } else {
        w = r * G + ((r & 1) ? (G - 1 - c) : c);
        if (w >= p.n_items) return false;
    }
    int qb;
    if (CAUSAL) {  // heaviest blocks first
        const int bh_count = p.B * p.Hq;
        it.bh = w % bh_count;
        qb = p.n_qblocks - 1 - w / bh_count;
    } else {  // head by head
        it.bh = w / p.n_qblocks;
        qb = w % p.n_qblocks;
    }
    it.b = it.bh / p.Hq;
    it.h = it.bh % p.Hq;
    it.hk = it.h / (p.Hq / p.Hkv);
    it.q0 = 2 * qb + (half > 0 ? 1 : 0);
    it.nk0 = CAUSAL ? min(2 * qb + 1, p.nblk) : p.nblk;
    it.nk1 = CAUSAL ? min(2 * qb + 2, p.nblk) : (half >= 0 ? 0 : p.nblk);
    it.nkv = max(it.nk0, it.nk1);
    return true;
}

// The FP8 forward: the persistent two-tile schedule of attn_fwd_kernel (two
// 128-row query tiles per item sharing every K/V tile, the two softmax
// warpgroups taking strict turns for the exp2 pass), with E4M3 operands and P
// through shared memory. Because P does not live in the S columns, S_t(j+1)
// is issued as soon as the softmax has read S_t(j) into registers and is
// computed while the softmax works on tile j: each tile's chain is its
// softmax alone.
//   warps 0-3 / 4-7  softmax and epilogue of query tile 0 / 1 (thread = row)
//   warps 8, 9       MMA issuers (tcgen05.mma kind::f8f6f4, both operands
//                    K-major in 128-byte-swizzled shared memory):
//                    S_t = Q8_t K8_j^T into TMEM, O_t += P8_t V8_j
//   warps 10, 11     TMA producers: Q tiles, then K_j and V^T_j tiles (16 KB
//                    each) into an 8-slot ring, one thread per tile of a pair
template <bool CAUSAL>
__global__ void __launch_bounds__(384, 1)
    attn_fwd_fp8_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_vt, const Fp8Params p) {
    using C = Fp8Cfg;
    constexpr int TILE = C::TILE, SLOTS = C::SLOTS, BM = C::BM, BN = C::BN;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = smem;                    // [2]
    uint8_t* sKV = sQ + C::TILES * TILE;   // [SLOTS]
    uint8_t* sP = sKV + SLOTS * TILE;      // [2] P of query tile t, 128 rows of 128 keys
    uint8_t* sO = sP + C::TILES * TILE;    // [8 warps][32 rows][64 bf16] epilogue staging
    uint64_t* bars = reinterpret_cast<uint64_t*>(sO + 8 * C::STAGE_O_BYTES);
    uint64_t* q_full = bars;                   // [2] Q tile t loaded
    uint64_t* q_empty = q_full + 2;            // [2] last S of Q tile t's buffer done
    uint64_t* slot_full = q_empty + 2;         // [SLOTS]
    uint64_t* slot_empty = slot_full + SLOTS;  // [SLOTS] released by both tiles' MMAs
    uint64_t* s_full = slot_empty + SLOTS;     // [2] S_t complete
    uint64_t* s_free = s_full + 2;             // [2] S_t read into registers (4 warp arrivals)
    uint64_t* p_full = s_free + 2;             // [2] P_t written (4 warp arrivals)
    uint64_t* pv_done = p_full + 2;            // [2] a P V product of tile t complete
    uint64_t* o_free = pv_done + 2;            // [2] epilogue has read O_t (4 warp arrivals)
    uint64_t* turn = o_free + 2;               // [2] softmax ping-pong (4 warp arrivals)
    uint64_t* drain = turn + 2;                // [2]
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 2);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int t = 0; t < 2; ++t) {
            mbar_init(&q_full[t], 1);
            mbar_init(&q_empty[t], 1);
            mbar_init(&s_full[t], 1);
            mbar_init(&s_free[t], 4);
            mbar_init(&p_full[t], 4);
            mbar_init(&pv_done[t], 1);
            mbar_init(&o_free[t], 4);
            mbar_init(&turn[t], 4);
            mbar_init(&drain[t], 1);
        }
        for (int i = 0; i < SLOTS; ++i) {
            mbar_init(&slot_full[i], 1);
            mbar_init(&slot_empty[i], 2);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 8) {
        tmem_alloc(tmem_holder, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    grid_dep_wait();  // the previous kernel's writes are visible from here on

    if (warp >= 10) {
        // ------------------------------------------------------ producers ---
        // K/V load g (K_j, V^T_j of an item are loads base + 2j, base + 2j + 1) and
        // Q tile t go to producer g % 2 and t % 2.
        if (lane == 0) {
            const int me = warp - 10;
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_vt);
            bool ok = true;
            int g = 0;
            int nq[2] = {0, 0};  // Q tile loads issued per buffer
            Fp8Item item;
            for (int r = 0; ok && fp8_item<CAUSAL>(p, r, item); ++r) {
                const int zq = item.b * p.Hq + item.h, zkv = item.b * p.Hkv + item.hk;
                auto issue_kv = [&](int i) -> bool {
                    const int gi = g + i;
                    if ((gi & 1) != me) return true;
                    const int slot = gi % SLOTS, use = gi / SLOTS;
                    if (use > 0 && !mbar_wait_park(&slot_empty[slot], (use - 1) & 1, abort_flag)) return false;
                    mbar_arrive_expect_tx(&slot_full[slot], TILE);
                    if (i & 1) tma_load_3d(sKV + slot * TILE, &tm_vt, &slot_full[slot], (i >> 1) * BN, 0, zkv);
                    else tma_load_3d(sKV + slot * TILE, &tm_k, &slot_full[slot], 0, (i >> 1) * BN, zkv);
                    return true;
                };
                auto issue_q = [&](int t) -> bool {
                    if ((t & 1) != me || (t == 1 && item.nk1 == 0)) return true;
                    if (nq[t] > 0 && !mbar_wait_park(&q_empty[t], (nq[t] - 1) & 1, abort_flag)) return false;
                    mbar_arrive_expect_tx(&q_full[t], TILE);
                    tma_load_3d(sQ + t * TILE, &tm_q, &q_full[t], 0, (item.q0 + t) * BM, zq);
                    ++nq[t];
                    return true;
                };
                ok = issue_q(0) && issue_kv(0) && issue_kv(1) && issue_q(1);
                for (int i = 2; ok && i < 2 * item.nkv; ++i) ok = issue_kv(i);
                g += 2 * item.nkv;
            }
            // Every load of this CTA is issued: the next kernel in the stream may be
            // scheduled (it waits for this grid's completion before reading memory).
            grid_dep_launch();
            // Let every copy in flight land before the CTA can exit.
            if (nq[me] > 0) mbar_wait(&q_full[me], (nq[me] - 1) & 1, nullptr);
            for (int i = max(0, g - SLOTS); i < g; ++i)
                if ((i & 1) == me) mbar_wait(&slot_full[i % SLOTS], (i / SLOTS) & 1, nullptr);
        }
    } else if (warp >= 8) {
        // ---------------------------------------------------- MMA issuers ---
        const int t = warp - 8;
        if (lane == 0) {
            // E4M3 x E4M3 -> F32, both operands K-major: the kind::f8f6f4 format
            // code of E4M3 is 0, so the descriptor bits match make_idesc's
            constexpr uint32_t idesc = make_idesc(128, 128, 0, 0, 0);
            const uint32_t s_tmem = tmem + t * 256, o_tmem = s_tmem + 128;
            const uint32_t q_addr = smem_addr(sQ + t * TILE), kv_addr = smem_addr(sKV), p_addr = smem_addr(sP + t * TILE);
            bool ok = true;
            int g = 0;
            uint32_t ns = 0, np = 0;  // S_t issued, P_t consumed: counted across items
            // S_t = Q_t K_j^T once the previous S_t has been read by the softmax
            auto issue_s = [&](int ik, bool solo_tile) -> bool {
                if (!mbar_wait(&slot_full[ik % SLOTS], (ik / SLOTS) & 1, abort_flag)) return false;
                if (ns > 0 && !mbar_wait(&s_free[t], (ns - 1) & 1, abort_flag)) return false;
                tc_fence_after();
                const uint32_t k_addr = kv_addr + (ik % SLOTS) * TILE;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)  // 32 bytes = 32 elements of K per MMA
                    mma_f8_ss(s_tmem, make_sdesc_sw128(q_addr + kk * 32, 16, 1024),
                              make_sdesc_sw128(k_addr + kk * 32, 16, 1024), idesc, kk > 0 ? 1u : 0u);
                tc_commit(&s_full[t]);
                if (solo_tile) mbar_arrive(&slot_empty[ik % SLOTS]);
                tc_commit(&slot_empty[ik % SLOTS]);
                ++ns;
                return true;
            };
            int nit = 0;  // items this tile took part in
            Fp8Item item;
            for (int r = 0; ok && fp8_item<CAUSAL>(p, r, item); ++r) {
                const int nk = t ? item.nk1 : item.nk0;
                // a K/V tile only this tile reads (tile 1's causal diagonal, or every
                // tile of a half item) takes both of the slot's releases
                auto solo = [&](int j) { return t ? j >= item.nk0 : j >= item.nk1; };
                if (nk == 0) {
                    g += 2 * item.nkv;
                    continue;
                }
                ok = mbar_wait(&q_full[t], nit & 1, abort_flag) && issue_s(g, solo(0));
                if (ok && nk == 1) tc_commit(&q_empty[t]);
                for (int j = 0; ok && j < nk; ++j) {
                    // S_t(j+1) goes ahead of P V(j): it runs while the softmax works on P_t(j)
                    if (j + 1 < nk) {
                        ok = issue_s(g + 2 * (j + 1), solo(j + 1));
                        if (!ok) break;
                        if (j + 1 == nk - 1) tc_commit(&q_empty[t]);  // Q_t buffer free after its last S
                    }
                    const int iv = g + 2 * j + 1;
                    ok = mbar_wait(&slot_full[iv % SLOTS], (iv / SLOTS) & 1, abort_flag) &&
                         (j > 0 || nit == 0 || mbar_wait(&o_free[t], (nit - 1) & 1, abort_flag)) &&
                         mbar_wait_spin(&p_full[t], np & 1, abort_flag);
                    if (!ok) break;
                    ++np;
                    tc_fence_after();
                    const uint32_t v_addr = kv_addr + (iv % SLOTS) * TILE;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_f8_ss(o_tmem, make_sdesc_sw128(p_addr + kk * 32, 16, 1024),
                                  make_sdesc_sw128(v_addr + kk * 32, 16, 1024), idesc, (j > 0 || kk > 0) ? 1u : 0u);
                    tc_commit(&pv_done[t]);
                    if (solo(j)) mbar_arrive(&slot_empty[iv % SLOTS]);
                    tc_commit(&slot_empty[iv % SLOTS]);
                }
                g += 2 * item.nkv;
                ++nit;
            }
            // Every MMA must be complete before TMEM is released.
            tc_commit(&drain[t]);
            mbar_wait(&drain[t], 0, nullptr);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------- softmax ----
        const int t = warp >> 2;
        const int quad = warp & 3;
        const int row = quad * 32 + lane;
        const uint32_t s_addr = tmem + t * 256 + (uint32_t(quad * 32) << 16);
        const uint32_t o_addr = s_addr + 128;
        bool ok = true;
        uint32_t ns = 0, nturn = 0, npv = 0;  // phases consumed, counted across items
        Fp8Item item;
        for (int r = 0; ok && fp8_item<CAUSAL>(p, r, item); ++r) {
            const int nk = t ? item.nk1 : item.nk0;
            if (nk == 0) continue;
            const int q128 = item.q0 + t;  // this query tile in 128-row units
            const int kvp = item.b * p.Hkv + item.hk;
            const float sq = q128 < p.nblk ? p.sq[static_cast<size_t>(item.bh) * p.nblk + q128] : 1.f;
            const float* skp = p.sk + static_cast<size_t>(kvp) * p.nblk;
            const int q_row = q128 * BM + row;
            float m_used = -INFINITY, l = 0.f;
            float sk_j = skp[0];
            for (int j = 0; j < nk; ++j) {
                const bool w1 = mbar_wait(&s_full[t], ns & 1, abort_flag);
                if (!__all_sync(0xffffffffu, w1)) { ok = false; break; }
                ++ns;
                tc_fence_after();
                uint32_t sr[128];
                tmem_ld64(s_addr, reinterpret_cast<uint32_t(&)[64]>(sr[0]));
                tmem_ld64(s_addr + 64, reinterpret_cast<uint32_t(&)[64]>(sr[64]));
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&s_free[t]);  // S_t(j+1) may overwrite S_t now
                // scores in log2 units: S8 x s_q x s_k(j) x scale x log2(e), c > 0
                const float c = p.scale_log2 * sq * sk_j;
                sk_j = j + 1 < nk ? skp[j + 1] : 0.f;  // loaded a key tile ahead
                int lim = BN;  // visible keys of this tile for this row: [0, lim)
                if (CAUSAL && j == q128) lim = row + 1;
                if (!CAUSAL && j * BN + BN > p.N) lim = p.N - j * BN;
                const bool full = __all_sync(0xffffffffu, lim == BN);
                if (!full) {
#pragma unroll
                    for (int i = 0; i < 128; ++i)
                        if (i >= lim) sr[i] = 0xff800000u;  // -inf: exp2 gives 0
                }
                const float m_tile = fp8_row_max(sr) * c;
                const bool need = m_tile > m_used + 8.f;  // P <= 2^8 between rescales, inside E4M3
                float factor = 1.f;
                if (need) {
                    factor = ex2_approx(m_used - m_tile);
                    m_used = m_tile;
                }
                // the two softmax warpgroups take turns for the exp2 pass (tile 1's extra
                // causal key tile, its diagonal, takes no turn), as in attn_fwd_kernel
                // (a half item has no tile 1: tile 0 only waits for the hand-over
                // left from the item before)
                const bool paired = item.nk1 > 0;
                const bool my_turn_wait = (t == 0) ? (paired ? (r > 0 || j > 0) : (r > 0 && j == 0)) : (j < item.nk0);
                if (my_turn_wait) {
                    const bool wt = mbar_wait(&turn[t], nturn & 1, abort_flag);
                    if (!__all_sync(0xffffffffu, wt)) { ok = false; break; }
                    ++nturn;
                }
                const float2 cc2 = make_float2(c, c), negm2 = make_float2(-m_used, -m_used);
                float2 rsum[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) rsum[k] = make_float2(0.f, 0.f);
                uint32_t pk[32];
                if (full) fp8_exp_row<kFp8PolyPairs>(sr, cc2, negm2, rsum, pk);
                else fp8_exp_row<0>(sr, cc2, negm2, rsum, pk);
                // pass the turn on (tile 0 to tile 1 of the same key tile; tile 1 back
                // after each key tile it shares with tile 0)
                const bool hand_over = (t == 0) ? paired : (j < item.nk0);
                if (hand_over && lane == 0) mbar_arrive(&turn[1 - t]);
                const float2 rs = fadd2(fadd2(rsum[0], rsum[1]), fadd2(rsum[2], rsum[3]));
                l = l * factor + (rs.x + rs.y);
                // P V(j - 1) must be complete: it still reads the P buffer, and O_t must
                // hold it before a rescale
                if (j >= 1) {
                    const bool w3 = mbar_wait(&pv_done[t], npv & 1, abort_flag);
                    if (!__all_sync(0xffffffffu, w3)) { ok = false; break; }
                    ++npv;
                }
                if (j >= 1 && __any_sync(0xffffffffu, factor != 1.f)) {
                    tc_fence_after();
#pragma unroll
                    for (int cch = 0; cch < 4; ++cch) {
                        uint32_t ov[32];
                        tmem_ld32(o_addr + cch * 32, ov);
#pragma unroll
                        for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * factor);
                        tmem_st32(o_addr + cch * 32, ov);
                    }
                    tmem_st_wait();
                }
                // P row into the 128-byte-swizzled K-major tile: 16-byte chunk cc of
                // row r sits at chunk position cc ^ (r & 7)
                uint8_t* prow = sP + t * TILE + row * 128;
#pragma unroll
                for (int cc = 0; cc < 8; ++cc)
                    *reinterpret_cast<uint4*>(prow + ((cc ^ (row & 7)) << 4)) =
                        make_uint4(pk[4 * cc], pk[4 * cc + 1], pk[4 * cc + 2], pk[4 * cc + 3]);
                fence_proxy_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&p_full[t]);
            }
            if (!ok) break;
            // Epilogue: O_t holds every P V product once the last one is complete.
            {
                const bool w2 = mbar_wait(&pv_done[t], npv & 1, abort_flag);
                if (!__all_sync(0xffffffffu, w2)) { ok = false; break; }
                ++npv;
            }
            tc_fence_after();
            const float f = p.sv[static_cast<size_t>(kvp) * p.nblk] / l;
            uint8_t* stage = sO + warp * C::STAGE_O_BYTES;
            const int row0 = q128 * BM + quad * 32;  // first row of this warp
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                // this lane's row, columns [64*half, 64*half + 64): 128 bytes as 8
                // chunks of 16; chunk i of row r sits at slot i ^ (r & 7)
#pragma unroll
                for (int c2 = 0; c2 < 2; ++c2) {
                    const int cch = half * 2 + c2;
                    uint32_t r3[32];
                    tmem_ld32(o_addr + cch * 32, r3);
                    if (cch == 3) {
                        // O_t is in registers: the next item's first P V may overwrite it
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&o_free[t]);
                    }
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int chunk = c2 * 4 + i;
                        const uint4 v4 = make_uint4(
                            pack_bf16x2(__uint_as_float(r3[8 * i + 0]) * f, __uint_as_float(r3[8 * i + 1]) * f),
                            pack_bf16x2(__uint_as_float(r3[8 * i + 2]) * f, __uint_as_float(r3[8 * i + 3]) * f),
                            pack_bf16x2(__uint_as_float(r3[8 * i + 4]) * f, __uint_as_float(r3[8 * i + 5]) * f),
                            pack_bf16x2(__uint_as_float(r3[8 * i + 6]) * f, __uint_as_float(r3[8 * i + 7]) * f));
                        *reinterpret_cast<uint4*>(stage + lane * 128 + ((chunk ^ (lane & 7)) << 4)) = v4;
                    }
                }
                __syncwarp();
                // read back: lane = 8 * (row within a group of 4) + chunk, 4 rows per store
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const int rr = 4 * k + (lane >> 3), chunk = lane & 7;
                    const uint4 v4 = *reinterpret_cast<const uint4*>(stage + rr * 128 + ((chunk ^ (rr & 7)) << 4));
                    if (row0 + rr < p.N)
                        *reinterpret_cast<uint4*>(p.o + (static_cast<size_t>(item.bh) * p.N + row0 + rr) * 128 +
                                                  half * 64 + chunk * 8) = v4;
                }
                __syncwarp();
            }
            if (q_row < p.N)
                p.lse[static_cast<size_t>(item.bh) * p.N + q_row] = (m_used + log2f(l)) * 0.69314718055994530942f;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 8) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

}  // namespace eab
