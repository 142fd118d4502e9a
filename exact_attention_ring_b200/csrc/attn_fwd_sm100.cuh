// Prefill forward pass on sm_100a: O = softmax(scale * Q K^T) V and the per-row
// log-sum-exp, one 128-row query tile per CTA.
//
// The method is the tiled online softmax of "1-Flash-Attention.md" (sections
// "Tiling（分块）技术", "递归计算softmax"): a query tile stays on chip while key /
// value tiles stream past it; per row a running max m and denominator l are
// kept, the accumulator is rescaled when the max moves, and O is divided by l
// once at the end (FlashAttention V2 page: fewer non-matmul operations). Loop
// order is the V2 one (query tile outer, key/value tiles inner).
//
// B200 mapping (warp-specialised, 192 threads):
//   warp 0    TMA producer: the Q tile once, then K_j and V_j tiles into a ring
//             of shared-memory slots guarded by full/empty mbarriers.
//   warp 1    MMA issuer (one thread): S_j = Q K_j^T with tcgen05.mma into one of
//             two TMEM score buffers, and O += P_j V_j with P read from TMEM.
//             Completion is signalled with tcgen05.commit onto mbarriers.
//   warps 2-5 softmax: one thread per query row (TMEM lane). Reads S_j, applies
//             the causal / ragged-tail mask, tracks the running max in log2
//             units (exp2 with scale*log2(e) folded into one FMA), rescales O in
//             TMEM only when the max grows by more than 2^8 (lazy rescale), writes
//             P_j as bf16 over the S_j columns, and finally normalises O.
// TMEM columns: S buffer 0 [0,128), S buffer 1 [128,256), O [256, 256+D).
// Shared memory: Q tile + SLOTS key/value tiles, all 128-byte swizzled as the
// tcgen05 K-major (Q, K) and MN-major (V) operand layouts expect.
#pragma once

#include "sm100_ptx.cuh"

namespace eab {

struct FwdParams {
    __nv_bfloat16* o;  // [B, Hq, N, D]
    float* lse;        // [B, Hq, N]
    int B, Hq, Hkv, N;
    int n_qtiles;
    float scale_log2;  // scale * log2(e)
};

template <int D>
struct FwdCfg {
    static constexpr int BM = 128;                 // query rows per tile (= TMEM lanes)
    static constexpr int BN = 128;                 // keys per tile
    static constexpr int CHUNKS = D / 64;          // 64-element (128-byte) swizzle chunks per row
    static constexpr int Q_BYTES = BM * D * 2;
    static constexpr int TILE_BYTES = BN * D * 2;  // one K or V tile
    static constexpr int SLOTS = (D == 128) ? 6 : 10;
    static constexpr int NUM_THREADS = 192;
    static constexpr int NUM_BARRIERS = 1 + 2 * SLOTS + 2 + 2 + 1 + 1;
    static constexpr int SMEM_BYTES = 1024 + Q_BYTES + SLOTS * TILE_BYTES + NUM_BARRIERS * 8 + 16;
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t O_COL = 256;
    static constexpr float RESCALE_THRESHOLD = 8.0f;  // log2 units: P <= 2^8 between rescales
};

template <int D, bool CAUSAL>
__global__ void __launch_bounds__(192, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
    using C = FwdCfg<D>;
    constexpr int BM = C::BM, BN = C::BN, SLOTS = C::SLOTS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = smem;
    uint8_t* sKV = smem + C::Q_BYTES;
    uint64_t* bars = reinterpret_cast<uint64_t*>(sKV + SLOTS * C::TILE_BYTES);
    uint64_t* q_full = bars;
    uint64_t* slot_full = bars + 1;
    uint64_t* slot_empty = slot_full + SLOTS;
    uint64_t* s_full = slot_empty + SLOTS;  // [2]
    uint64_t* p_full = s_full + 2;          // [2]
    uint64_t* o_done = p_full + 2;
    uint64_t* drain = o_done + 1;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // Work tile: heaviest causal query tiles are scheduled first.
    const int bh_count = p.B * p.Hq;
    const int rank = blockIdx.x / bh_count;
    const int bh = blockIdx.x % bh_count;
    const int qt = CAUSAL ? (p.n_qtiles - 1 - rank) : rank;
    const int b = bh / p.Hq, h = bh % p.Hq;
    const int hk = h / (p.Hq / p.Hkv);
    const int n_kv_tiles = (p.N + BN - 1) / BN;
    const int nk = CAUSAL ? min(qt + 1, n_kv_tiles) : n_kv_tiles;

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int i = 0; i < SLOTS; ++i) {
            mbar_init(&slot_full[i], 1);
            mbar_init(&slot_empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s_full[i], 1);
            mbar_init(&p_full[i], 128);
        }
        mbar_init(o_done, 1);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    if (warp == 0) {
        // ------------------------------------------------------ producer ----
        if (lane == 0) {
            const int zq = b * p.Hq + h, zkv = b * p.Hkv + hk;
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            mbar_arrive_expect_tx(q_full, C::Q_BYTES);
#pragma unroll
            for (int c = 0; c < C::CHUNKS; ++c) tma_load_3d(sQ + c * BM * 128, &tm_q, q_full, c * 64, qt * BM, zq);
            int issued = 0;
            for (int i = 0; i < 2 * nk; ++i) {
                const int slot = i % SLOTS, use = i / SLOTS;
                if (use > 0 && !mbar_wait(&slot_empty[slot], (use - 1) & 1, abort_flag)) break;
                const CUtensorMap* tm = (i & 1) ? &tm_v : &tm_k;
                uint8_t* dst = sKV + slot * C::TILE_BYTES;
                mbar_arrive_expect_tx(&slot_full[slot], C::TILE_BYTES);
#pragma unroll
                for (int c = 0; c < C::CHUNKS; ++c)
                    tma_load_3d(dst + c * BN * 128, tm, &slot_full[slot], c * 64, (i >> 1) * BN, zkv);
                issued = i + 1;
            }
            // Let every copy in flight land before the CTA can exit.
            mbar_wait(q_full, 0, nullptr);
            for (int i = max(0, issued - SLOTS); i < issued; ++i)
                mbar_wait(&slot_full[i % SLOTS], (i / SLOTS) & 1, nullptr);
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA -----
        if (lane == 0) {
            constexpr uint32_t idesc_qk = make_idesc_bf16(BM, BN, 0, 0);
            constexpr uint32_t idesc_pv = make_idesc_bf16(BM, D, 0, 1);
            const uint32_t q_addr = smem_addr(sQ), kv_addr = smem_addr(sKV);
            bool ok = mbar_wait(q_full, 0, abort_flag);
            auto issue_s = [&](int j) -> bool {
                const int i = 2 * j, slot = i % SLOTS;
                if (!mbar_wait(&slot_full[slot], (i / SLOTS) & 1, abort_flag)) return false;
                tc_fence_after();
                const uint32_t k_addr = kv_addr + slot * C::TILE_BYTES;
                const uint32_t d_tmem = tmem + (j & 1) * 128;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t koff = (kk & 3) * 32;  // 16 elements = 32 bytes inside the swizzle row
                    const uint64_t ad = make_sdesc_sw128(q_addr + (kk >> 2) * BM * 128 + koff, 16, 1024);
                    const uint64_t bd = make_sdesc_sw128(k_addr + (kk >> 2) * BN * 128 + koff, 16, 1024);
                    mma_ss(d_tmem, ad, bd, idesc_qk, kk > 0 ? 1u : 0u);
                }
                tc_commit(&s_full[j & 1]);
                tc_commit(&slot_empty[slot]);
                return true;
            };
            if (ok) ok = issue_s(0);
            if (ok && nk > 1) ok = issue_s(1);
            for (int j = 0; ok && j < nk; ++j) {
                if (!mbar_wait(&p_full[j & 1], (j >> 1) & 1, abort_flag)) break;
                const int i = 2 * j + 1, slot = i % SLOTS;
                if (!mbar_wait(&slot_full[slot], (i / SLOTS) & 1, abort_flag)) break;
                tc_fence_after();
                const uint32_t v_addr = kv_addr + slot * C::TILE_BYTES;
                const uint32_t a_tmem = tmem + (j & 1) * 128;
#pragma unroll
                for (int kk = 0; kk < BN / 16; ++kk) {
                    // V tile as the MN-major B operand: 16 keys = 2048 bytes per step;
                    // LBO = distance between the 64-column chunks of the tile.
                    const uint64_t bd = make_sdesc_sw128(v_addr + kk * 16 * 128, BN * 128, 1024);
                    mma_ts(tmem + C::O_COL, a_tmem + kk * 8, bd, idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
                }
                tc_commit(o_done);
                tc_commit(&slot_empty[slot]);
                if (j + 2 < nk) ok = issue_s(j + 2);
            }
            // Every MMA must be complete before TMEM is released.
            tc_commit(drain);
            mbar_wait(drain, 0, nullptr);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------ softmax -----
        const int quad = warp & 3;  // TMEM lane quadrant this warp may access
        const int row = quad * 32 + lane;
        const int grow = qt * BM + row;
        const uint32_t lane_base = tmem + (uint32_t(quad * 32) << 16);
        const float c2 = p.scale_log2;
        float m_used = -INFINITY, l = 0.f;
        bool ok = true;
        for (int j = 0; j < nk; ++j) {
            const bool w = mbar_wait(&s_full[j & 1], (j >> 1) & 1, abort_flag);
            if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
            tc_fence_after();
            const uint32_t s_addr = lane_base + (j & 1) * 128;
            float s[BN];
#pragma unroll
            for (int c = 0; c < BN / 32; ++c) {
                uint32_t r[32];
                tmem_ld32(s_addr + c * 32, r);
#pragma unroll
                for (int i = 0; i < 32; ++i) s[c * 32 + i] = __uint_as_float(r[i]);
            }
            const int kv0 = j * BN;
            if (CAUSAL && j == qt) {
#pragma unroll
                for (int i = 0; i < BN; ++i)
                    if (i > row) s[i] = -INFINITY;
            } else if (!CAUSAL && kv0 + BN > p.N) {
                const int lim = p.N - kv0;
#pragma unroll
                for (int i = 0; i < BN; ++i)
                    if (i >= lim) s[i] = -INFINITY;
            }
            float mx = s[0];
#pragma unroll
            for (int i = 1; i < BN; ++i) mx = fmaxf(mx, s[i]);
            const float m_tile = mx * c2;
            const bool need = m_tile > m_used + C::RESCALE_THRESHOLD;
            float factor = 1.f;
            if (need) {
                factor = ex2_approx(m_used - m_tile);
                m_used = m_tile;
            }
            l *= factor;
            const float neg_m = -m_used;
            float rs = 0.f;
            uint32_t pk[BN / 2];
#pragma unroll
            for (int i = 0; i < BN / 2; ++i) {
                const float p0 = ex2_approx(fmaf(s[2 * i], c2, neg_m));
                const float p1 = ex2_approx(fmaf(s[2 * i + 1], c2, neg_m));
                rs += p0 + p1;
                pk[i] = pack_bf16x2(p0, p1);
            }
            l += rs;
            if (j > 0) {
                // Every PV completion is awaited in order, so the parity wait on
                // o_done can never alias a phase two completions back. PV_{j-1}
                // was issued a whole tile ago, so this rarely stalls.
                const bool w2 = mbar_wait(o_done, (j - 1) & 1, abort_flag);
                if (!__all_sync(0xffffffffu, w2)) { ok = false; break; }
                if (__any_sync(0xffffffffu, need)) {
                    tc_fence_after();
#pragma unroll
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t r[32];
                        tmem_ld32(lane_base + C::O_COL + c * 32, r);
#pragma unroll
                        for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * factor);
                        tmem_st32(lane_base + C::O_COL + c * 32, r);
                    }
                }
            }
#pragma unroll
            for (int c = 0; c < BN / 64; ++c) {
                uint32_t chunk[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) chunk[i] = pk[c * 32 + i];
                tmem_st32(s_addr + c * 32, chunk);
            }
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(&p_full[j & 1]);
        }
        if (ok) {
            const bool w = mbar_wait(o_done, (nk - 1) & 1, abort_flag);
            if (__all_sync(0xffffffffu, w)) {
                tc_fence_after();
                const float inv_l = 1.f / l;
                __nv_bfloat16* orow = p.o + (static_cast<size_t>(bh) * p.N + grow) * D;
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t r[32];
                    tmem_ld32(lane_base + C::O_COL + c * 32, r);
                    uint32_t pk[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        pk[i] = pack_bf16x2(__uint_as_float(r[2 * i]) * inv_l, __uint_as_float(r[2 * i + 1]) * inv_l);
                    if (grow < p.N) {
                        uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
                    }
                }
                if (grow < p.N)
                    p.lse[static_cast<size_t>(bh) * p.N + grow] = (m_used + log2f(l)) * 0.69314718055994530942f;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

}  // namespace eab
