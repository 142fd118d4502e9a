// Backward pass on sm_100a: dQ, dK, dV of exact attention from the forward's
// O and LSE, recomputing P tile by tile.
//
// The forward pass keeps only O and the per-row log-sum-exp, so P is rebuilt
// from S = scale Q K^T and the LSE (FlashAttention V2 page, opening paragraph:
// tiling plus recomputation, the N x N matrices never written out; Flash
// Attention notes, "使用注意事项": the backward pass accumulates the softmax
// terms in fp32). With
// dP = dO V^T, Delta_i = sum_t dO_it O_it = sum_j P_ij dP_ij and
// dS = P o (dP - Delta):
//   dV = P^T dO,   dK = scale dS^T Q,   dQ = scale dS K.
// Three launches:
//   bwd_delta_kernel        Delta per row (one warp per row, HBM-bound);
//   bwd_tile_kernel, DKDV   one 128-key tile of one (batch, KV head) per block:
//                           for every query head of the group and every query
//                           tile that sees the keys, S^T = K Q^T and
//                           dP^T = V dO^T into TMEM, P^T and dS^T (bf16)
//                           written back over them by the element-wise warps
//                           (one thread per key), then dV += P^T dO and
//                           dK += dS^T Q with A from TMEM (scale applied to dK
//                           once, in the epilogue);
//   bwd_tile_kernel, !DKDV  one 128-row query tile of one (batch, query head)
//                           per block: S = Q K^T and dP = dO V^T per key tile,
//                           dS (bf16) over dP, dQ += dS K (then times scale).
// 320 threads each: warps 0-7 element-wise work and epilogue (thread = TMEM
// lane; warps w and w + 4 share lane quarter w and split its 128 columns in
// halves), warp 8 the MMA issuer, warp 9 the TMA producer. Within a step the
// element-wise pass reads S^T into registers at once, so the next step's S^T
// MMAs run while it computes P (as dP^T is completing) and dS; P and dS go
// back as bf16 over dP^T's columns, a quarter at a time, and are handed over
// in two halves of 64 columns: the accumulating MMAs of the first half run
// while the second half is computed. The next step's dP^T MMAs are issued
// after the accumulating MMAs that read P^T / dS^T from its columns, so the
// tensor pipe's issue order keeps them intact until read (as in the forward
// pass). Every wait is bounded. The dQ kernel needs nothing the dK/dV kernel
// writes: its blocks start as the dK/dV tail frees SMs and wait for that grid
// only before they exit.
#pragma once

#include "sm100_ptx.cuh"

namespace eab {

struct BwdParams {
    const __nv_bfloat16* o;     // [B, Hq, N, D]
    const __nv_bfloat16* dout;  // [B, Hq, N, D]
    const float* lse;           // [B, Hq, N]
    float* delta;               // [B, Hq, N] (written by bwd_delta_kernel)
    __nv_bfloat16* dq;          // [B, Hq, N, D]
    __nv_bfloat16* dk;          // [B, Hkv, N, D]
    __nv_bfloat16* dv;          // [B, Hkv, N, D]
    int B, Hq, Hkv, N;
    float scale, scale_log2;
};

template <int D>
struct BwdCfg {
    static constexpr int BT = 128;                 // rows of a query tile / keys of a key tile
    static constexpr int CHUNKS = D / 64;
    static constexpr int TILE_BYTES = BT * D * 2;  // one 128 x D bf16 tile
    static constexpr int NUM_THREADS = 320;
    // [fixed A, B tiles][2 buffers x 2 streamed tiles][lse/delta 2 x 2 x 128 floats][barriers]
    static constexpr int SMEM_USED = 1024 + 2 * TILE_BYTES + 4 * TILE_BYTES + 4 * BT * 4 + 16 * 8 + 16;
    // A block allocates all 512 TMEM columns, so two blocks must never share an
    // SM (the second would stall in tcgen05.alloc): ask for more than half of
    // the SM's shared memory.
    static constexpr int SMEM_BYTES = SMEM_USED > 120 * 1024 ? SMEM_USED : 120 * 1024;
    static constexpr uint32_t TMEM_COLS = 512;
};

// Delta_i = sum_t dO_it O_it: D / 8 threads per row, each with one 16-byte load
// of dO and of O (8 elements), the partial sums reduced across those threads.
template <int D>
__global__ void __launch_bounds__(256) bwd_delta_kernel(const BwdParams p, long long rows) {
    grid_dep_wait();  // the previous kernel's writes are visible from here on
    grid_dep_launch();
    constexpr int TPR = D / 8;  // threads per row (16 or 8)
    const long long row = static_cast<long long>(blockIdx.x) * (256 / TPR) + threadIdx.x / TPR;
    const int part = threadIdx.x % TPR;
    float acc = 0.f;
    if (row < rows) {
        const uint4 a = *reinterpret_cast<const uint4*>(p.dout + row * D + part * 8);
        const uint4 b = *reinterpret_cast<const uint4*>(p.o + row * D + part * 8);
        const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 af = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&aw[i]));
            const float2 bf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&bw[i]));
            acc += af.x * bf.x + af.y * bf.y;
        }
    }
#pragma unroll
    for (int off = TPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (row < rows && part == 0) p.delta[row] = acc;
}

// Shared skeleton of the two tile kernels. One block owns a fixed pair of
// tiles (A_fix, B_fix: K and V for dK/dV; Q and dO for dQ) and streams pairs of
// tiles (S_a, S_b: Q and dO; K and V) through two buffers. Per step:
//   X = A_fix S_a^T, then Y = B_fix S_b^T          (M = 128, N = 128, K = D)
//   element-wise: X into registers (X's columns are then free, and the MMA
//     issuer starts X of the next step), P = exp2(X scale log2e - lse log2e)
//     for the 128 columns, then per quarter of 32 columns G = P o (Y - Delta)
//     with P and G written back as bf16 pairs over that quarter of Y
//     (columns 32q .. 32q + 15 and 32q + 16 .. 32q + 31), announced per half
//   acc1 += P S_b, acc2 += G S_a                    (A from TMEM, B MN-major)
// The accumulating MMAs of the first half run while the second half is being
// computed; Y of the next step follows them. For dQ only acc2 (dS K) is kept
// (P is not written back). scale multiplies acc2 once, in the epilogue. Steps
// whose tile holds no masked element (off the causal diagonal, inside the
// sequence) skip the mask.
// TMEM: X [0, 128), Y [128, 256), acc1 [256, 256 + D), acc2 [256 + D, 256 + 2D).
template <int D, bool CAUSAL, bool DKDV>
__global__ void __launch_bounds__(320, 1)
    bwd_tile_kernel(const __grid_constant__ CUtensorMap tm_fa, const __grid_constant__ CUtensorMap tm_fb,
                    const __grid_constant__ CUtensorMap tm_sa, const __grid_constant__ CUtensorMap tm_sb,
                    const BwdParams p) {
    using C = BwdCfg<D>;
    constexpr int BT = C::BT;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sFA = smem;
    uint8_t* sFB = sFA + C::TILE_BYTES;
    uint8_t* sS = sFB + C::TILE_BYTES;  // [2 buffers][S_a, S_b]
    // [2 buffers][-lse log2e, -Delta][128]: per streamed query row (dK/dV only)
    float* sL = reinterpret_cast<float*>(sS + 4 * C::TILE_BYTES);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sL + 4 * BT);
    uint64_t* fix_full = bars;       // the fixed tiles loaded
    uint64_t* st_full = bars + 1;    // [2] streamed tiles of a buffer loaded
    uint64_t* st_empty = bars + 3;   // [2] streamed tiles of a buffer read by every MMA
    uint64_t* x_full = bars + 5;     // X complete
    uint64_t* y_full = bars + 6;     // Y complete
    uint64_t* pg_half = bars + 7;    // [2] P and G of a half written (its 4 warps)
    uint64_t* l_ready = bars + 9;    // [2] lse/Delta of a buffer staged (4 warp arrivals)
    uint64_t* l_free = bars + 11;    // [2] lse/Delta of a buffer read (8 warp arrivals)
    uint64_t* fin = bars + 13;       // every MMA done
    uint64_t* x_read = bars + 14;    // X in the element-wise warps' registers (8 warp arrivals)
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 15);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = p.Hq / p.Hkv;
    const int n_tiles = (p.N + BT - 1) / BT;
    // the fixed tile: key tile (dK/dV) or query tile (dQ). The grid is (planes,
    // tiles) and blocks start in the order of their linear index, planes
    // fastest: under the causal mask every plane's block with the most steps
    // starts before any block with fewer, so the last wave holds the shortest.
    const int tile = (DKDV || !CAUSAL) ? blockIdx.y : n_tiles - 1 - blockIdx.y;
    // fixed head (KV head for dK/dV, query head for dQ) and its batch
    const int b = blockIdx.x / (DKDV ? p.Hkv : p.Hq);
    const int hfix = blockIdx.x % (DKDV ? p.Hkv : p.Hq);
    // the streamed steps: dK/dV walks (query head of the group, query tile);
    // dQ walks key tiles. Causal: query tile >= key tile.
    const int t_lo = DKDV ? (CAUSAL ? tile : 0) : 0;
    const int t_hi = DKDV ? n_tiles : (CAUSAL ? tile + 1 : n_tiles);
    const int per_head = t_hi - t_lo;
    const int nsteps = DKDV ? G * per_head : per_head;

    if (threadIdx.x == 0) {
        mbar_init(fix_full, 2 * C::CHUNKS);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&st_full[i], 2 * C::CHUNKS);
            mbar_init(&st_empty[i], 1);
            mbar_init(&pg_half[i], 4);
            mbar_init(&l_ready[i], 4);
            mbar_init(&l_free[i], 8);
        }
        mbar_init(x_full, 1);
        mbar_init(y_full, 1);
        mbar_init(fin, 1);
        mbar_init(x_read, 8);
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
    // The dK/dV kernel waits for the previous kernel (Delta) here. The dQ kernel
    // reads nothing the dK/dV kernel writes, and it is scheduled only once every
    // dK/dV block has passed its own wait (its trigger follows it), so Delta is
    // complete by then: its blocks start on the SMs the dK/dV tail frees and wait
    // for the dK/dV grid only before they exit, which keeps the stream's order
    // of completion.
    if (DKDV) grid_dep_wait();

    // plane (batch * heads + head) and tile row of streamed step s
    auto step_src = [&](int s, int* plane, int* trow) {
        if (DKDV) {
            const int h = hfix * G + s / per_head;
            *plane = b * p.Hq + h;
            *trow = (t_lo + s % per_head) * BT;
        } else {
            *plane = b * p.Hkv + hfix / G;
            *trow = (t_lo + s) * BT;
        }
    };

    if (warp == 9) {
        // ------------------------------------------------------ producer ----
        if (lane == 0 && nsteps > 0) {
            constexpr uint32_t BOX = BT * 128;
            const int fplane = DKDV ? b * p.Hkv + hfix : b * p.Hq + hfix;
#pragma unroll
            for (int c = 0; c < C::CHUNKS; ++c) {
                mbar_arrive_expect_tx(fix_full, BOX);
                tma_load_3d(sFA + c * BOX, &tm_fa, fix_full, c * 64, tile * BT, fplane);
                mbar_arrive_expect_tx(fix_full, BOX);
                tma_load_3d(sFB + c * BOX, &tm_fb, fix_full, c * 64, tile * BT, fplane);
            }
            int s = 0;
            for (; s < nsteps; ++s) {
                const int bu = s & 1;
                if (s >= 2 && !mbar_wait(&st_empty[bu], ((s >> 1) - 1) & 1, abort_flag)) break;
                int plane, trow;
                step_src(s, &plane, &trow);
                uint8_t* dst = sS + bu * 2 * C::TILE_BYTES;
#pragma unroll
                for (int c = 0; c < C::CHUNKS; ++c) {
                    mbar_arrive_expect_tx(&st_full[bu], BOX);
                    tma_load_3d(dst + c * BOX, &tm_sa, &st_full[bu], c * 64, trow, plane);
                    mbar_arrive_expect_tx(&st_full[bu], BOX);
                    tma_load_3d(dst + C::TILE_BYTES + c * BOX, &tm_sb, &st_full[bu], c * 64, trow, plane);
                }
            }
            // Every load of this CTA is issued: the next kernel in the stream may be
            // scheduled (it waits for this grid's completion before reading memory).
            grid_dep_launch();
            // Let every copy in flight land before the CTA can exit.
            mbar_wait(fix_full, 0, nullptr);
            for (int i = max(0, s - 2); i < s; ++i) mbar_wait(&st_full[i & 1], (i >> 1) & 1, nullptr);
        }
    } else if (warp == 8) {
        // ---------------------------------------------------- MMA issuer ----
        if (lane == 0 && nsteps > 0) {
            constexpr uint32_t idesc_xy = make_idesc(BT, BT, 0, 0, ElemBf16::fmt);  // A, B K-major
            constexpr uint32_t idesc_acc = make_idesc(BT, D, 0, 1, ElemBf16::fmt);  // B MN-major
            const uint32_t tX = tmem, tY = tmem + 128, tA1 = tmem + 256, tA2 = tmem + 256 + D;
            const uint32_t fa = smem_addr(sFA), fb = smem_addr(sFB);
            // X(s) = A_fix S_a(s)^T into X's columns, once step s's tiles have landed
            auto issue_x = [&](int s) -> bool {
                const int bu = s & 1;
                if (!mbar_wait(&st_full[bu], (s >> 1) & 1, abort_flag)) return false;
                tc_fence_after();
                const uint32_t sa = smem_addr(sS + bu * 2 * C::TILE_BYTES);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t koff = (kk >> 2) * (BT * 128) + (kk & 3) * 32;
                    mma_ss(tX, make_sdesc_sw128(fa + koff, 16, 1024), make_sdesc_sw128(sa + koff, 16, 1024), idesc_xy,
                           kk > 0 ? 1u : 0u);
                }
                tc_commit(x_full);
                return true;
            };
            // Y(s) = B_fix S_b(s)^T into Y's columns (after X(s): its tiles have landed)
            auto issue_y = [&](int s) {
                const uint32_t sb = smem_addr(sS + (s & 1) * 2 * C::TILE_BYTES) + C::TILE_BYTES;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t koff = (kk >> 2) * (BT * 128) + (kk & 3) * 32;
                    mma_ss(tY, make_sdesc_sw128(fb + koff, 16, 1024), make_sdesc_sw128(sb + koff, 16, 1024), idesc_xy,
                           kk > 0 ? 1u : 0u);
                }
                tc_commit(y_full);
            };
            bool ok = mbar_wait(fix_full, 0, abort_flag) && issue_x(0);
            if (ok) issue_y(0);
            for (int s = 0; ok && s < nsteps; ++s) {
                const int bu = s & 1;
                const uint32_t sa = smem_addr(sS + bu * 2 * C::TILE_BYTES), sb = sa + C::TILE_BYTES;
                // X(s+1) as soon as the element-wise warps hold X(s) in registers: it
                // is computed while they work on step s
                if (s + 1 < nsteps) {
                    ok = mbar_wait_spin(x_read, s & 1, abort_flag) && issue_x(s + 1);
                    if (!ok) break;
                }
                // acc1 += P S_b (dV += P^T dO), acc2 += G S_a (dK += dS^T Q, or
                // dQ += dS K), 64 streamed rows per half as each half lands. P and G of
                // the 32 streamed rows 32q .. 32q + 31 sit in Y's columns 32q .. 32q + 15
                // and 32q + 16 .. 32q + 31.
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    ok = mbar_wait_spin(&pg_half[h], s & 1, abort_flag);
                    if (!ok) break;
                    tc_fence_after();
#pragma unroll
                    for (int kk = h * (BT / 32); kk < (h + 1) * (BT / 32); ++kk) {
                        const uint32_t acc = (s > 0 || kk > 0) ? 1u : 0u;
                        const uint32_t pcol = tY + 32 * (kk >> 1) + 8 * (kk & 1);
                        if (DKDV)
                            mma_ts(tA1, pcol, make_sdesc_sw128(sb + kk * 16 * 128, BT * 128, 1024), idesc_acc, acc);
                        mma_ts(tA2, pcol + 16, make_sdesc_sw128(sa + kk * 16 * 128, BT * 128, 1024), idesc_acc, acc);
                    }
                }
                if (!ok) break;
                tc_commit(&st_empty[bu]);
                // Y(s+1) over the P and G the accumulating MMAs above read: the tensor
                // pipe's issue order keeps them intact until read
                if (s + 1 < nsteps) issue_y(s + 1);
            }
            tc_commit(fin);
            mbar_wait(fin, 0, nullptr);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------- element-wise -----
        // warps w and w + 4 share TMEM lane quarter w: w < 4 takes columns
        // 0 .. 63 (half 0), w >= 4 columns 64 .. 127 (half 1) of the same rows
        const int quad = warp & 3, grp = warp >> 2;
        const int row = quad * 32 + lane;  // TMEM lane: key (dK/dV) or query row (dQ)
        const uint32_t lb = tmem + (uint32_t(quad * 32) << 16);
        const uint32_t tX = lb, tY = lb + 128, tA1 = lb + 256, tA2 = lb + 256 + D;
        const float2 c2 = make_float2(p.scale_log2, p.scale_log2);
        const float LOG2E = 1.4426950408889634f;
        const int fixed_pos = tile * BT + row;  // this thread's key (dK/dV) or query row (dQ)
        // dQ: this thread's own row's -lse log2e and -Delta (rows past the end: P = 0)
        float nl2_row = -INFINITY, ndl_row = 0.f;
        if (!DKDV && fixed_pos < p.N) {
            const size_t r = static_cast<size_t>(b * p.Hq + hfix) * p.N + fixed_pos;
            nl2_row = -p.lse[r] * LOG2E;
            ndl_row = -p.delta[r];
        }
        // dK/dV: -lse log2e and -Delta of the streamed query rows, staged in
        // shared memory one step ahead by warps 0-3 (each thread one row)
        auto stage_load = [&](int s, float* nl2, float* ndl) {
            int plane, trow;
            step_src(s, &plane, &trow);
            const int qr = trow + row;
            const size_t r = static_cast<size_t>(plane) * p.N + qr;
            *nl2 = qr < p.N ? -p.lse[r] * LOG2E : -INFINITY;
            *ndl = qr < p.N ? -p.delta[r] : 0.f;
        };
        auto stage_store = [&](int s, float nl2, float ndl) {
            float* lsb = sL + (s & 1) * 2 * BT;
            lsb[row] = nl2;
            lsb[BT + row] = ndl;
            __syncwarp();
            if (lane == 0) mbar_arrive(&l_ready[s & 1]);
        };
        const bool stager = DKDV && grp == 0;
        bool ok = nsteps > 0;
        float pre_nl2 = 0.f, pre_ndl = 0.f;
        if (stager && ok) {
            stage_load(0, &pre_nl2, &pre_ndl);
            stage_store(0, pre_nl2, pre_ndl);
        }
        const int c0 = 64 * grp;  // this warp's first column
        for (int s = 0; ok && s < nsteps; ++s) {
            int plane, trow;
            step_src(s, &plane, &trow);
            if (stager && s + 1 < nsteps) stage_load(s + 1, &pre_nl2, &pre_ndl);
            const float* lsb = sL + (s & 1) * 2 * BT;
            if (DKDV && !__all_sync(0xffffffffu, mbar_wait(&l_ready[s & 1], (s >> 1) & 1, abort_flag))) {
                ok = false;
                break;
            }
            // visible columns of this thread's row: lo <= col < hi
            // (dK/dV: query = trow + col >= key; dQ: key = trow + col <= query)
            const int hi = DKDV ? p.N - trow : (CAUSAL ? min(p.N, fixed_pos + 1) : p.N) - trow;
            const int lo = (DKDV && CAUSAL) ? fixed_pos - trow : 0;
            const bool need_mask = trow + BT > p.N || (CAUSAL && trow == tile * BT);
            if (!__all_sync(0xffffffffu, mbar_wait(x_full, s & 1, abort_flag))) {
                ok = false;
                break;
            }
            tc_fence_after();
            // this warp's half of X into registers: X's columns are then free for X(s+1)
            uint32_t xv[64];
            tmem_ld64(tX + c0, xv);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(x_read);
            // P of the 64 columns, in place
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const int col = c0 + 2 * i;
                const float2 nl2 = DKDV ? *reinterpret_cast<const float2*>(lsb + col) : make_float2(nl2_row, nl2_row);
                const float2 a = ffma2(make_float2(__uint_as_float(xv[2 * i]), __uint_as_float(xv[2 * i + 1])), c2, nl2);
                xv[2 * i] = __float_as_uint(ex2_approx(a.x));
                xv[2 * i + 1] = __float_as_uint(ex2_approx(a.y));
            }
            if (need_mask) {
#pragma unroll
                for (int i = 0; i < 64; ++i)
                    if (c0 + i < lo || c0 + i >= hi) xv[i] = 0u;
            }
            if (!__all_sync(0xffffffffu, mbar_wait(y_full, s & 1, abort_flag))) {
                ok = false;
                break;
            }
            tc_fence_after();
            // G = P (Y - Delta), 32 columns at a time; P and G of columns 32q .. 32q + 31
            // go back as bf16 pairs over Y's columns 32q .. 32q + 15 and 32q + 16 .. 32q + 31
#pragma unroll
            for (int q2 = 0; q2 < 2; ++q2) {
                const int q = 2 * grp + q2;
                uint32_t ys[32], pk[16], gk[16];
                tmem_ld32(tY + 32 * q, ys);
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int j = 32 * q2 + 2 * i;  // column inside this warp's half
                    const float2 ndl = DKDV ? *reinterpret_cast<const float2*>(lsb + BT + c0 + j)
                                            : make_float2(ndl_row, ndl_row);
                    const float2 t = fadd2(make_float2(__uint_as_float(ys[2 * i]), __uint_as_float(ys[2 * i + 1])), ndl);
                    const float2 pp = make_float2(__uint_as_float(xv[j]), __uint_as_float(xv[j + 1]));
                    const float2 g = fmul2(pp, t);
                    pk[i] = pack_bf16x2(pp.x, pp.y);
                    gk[i] = pack_bf16x2(g.x, g.y);
                }
                if (DKDV) tmem_st16(tY + 32 * q, pk);
                tmem_st16(tY + 32 * q + 16, gk);
            }
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&pg_half[grp]);
            if (DKDV) {
                __syncwarp();
                if (lane == 0) mbar_arrive(&l_free[s & 1]);
                if (stager && s + 1 < nsteps) {
                    // buffer (s + 1) & 1 was last read in step s - 1 (by both halves)
                    if (s >= 1 &&
                        !__all_sync(0xffffffffu, mbar_wait(&l_free[(s + 1) & 1], ((s - 1) >> 1) & 1, abort_flag))) {
                        ok = false;
                        break;
                    }
                    stage_store(s + 1, pre_nl2, pre_ndl);
                }
            }
        }
        // epilogue: the accumulators (dV, dK; or dQ) to bf16 rows of the output
        if (ok && __all_sync(0xffffffffu, mbar_wait(fin, 0, abort_flag))) {
            tc_fence_after();
            // the TMEM loads are warp-wide; only rows inside the sequence are stored
            const bool in_seq = fixed_pos < p.N;
            const size_t out_row =
                static_cast<size_t>(DKDV ? b * p.Hkv + hfix : b * p.Hq + hfix) * p.N + (in_seq ? fixed_pos : 0);
            // dK/dV: warps 0-3 write dV, warps 4-7 dK; dQ: each group half of the columns
            {
                const int which = DKDV ? grp : 1;
                __nv_bfloat16* dst = (DKDV ? (which == 0 ? p.dv : p.dk) : p.dq) + out_row * D;
                const uint32_t src = which == 0 ? tA1 : tA2;
                const float f = which == 0 ? 1.f : p.scale;  // dK, dQ carry the scale
                const int c_lo = DKDV ? 0 : grp * (D / 64), c_hi = DKDV ? D / 32 : (grp + 1) * (D / 64);
#pragma unroll
                for (int c = c_lo; c < c_hi; ++c) {
                    uint32_t r3[32];
                    tmem_ld32(src + c * 32, r3);
                    if (in_seq) {
#pragma unroll
                        for (int i = 0; i < 32; i += 8)
                            *reinterpret_cast<uint4*>(dst + c * 32 + i) = make_uint4(
                                pack_bf16x2(__uint_as_float(r3[i]) * f, __uint_as_float(r3[i + 1]) * f),
                                pack_bf16x2(__uint_as_float(r3[i + 2]) * f, __uint_as_float(r3[i + 3]) * f),
                                pack_bf16x2(__uint_as_float(r3[i + 4]) * f, __uint_as_float(r3[i + 5]) * f),
                                pack_bf16x2(__uint_as_float(r3[i + 6]) * f, __uint_as_float(r3[i + 7]) * f));
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 4) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
    if (!DKDV) grid_dep_wait();
}

}  // namespace eab
