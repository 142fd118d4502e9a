// Split-KV single-query decode on the tensor cores, and the log-sum-exp
// weighted combine.
//
// Flash-Decoding (FlashAttention V2 page): for one query token the key/value
// range is split across thread blocks so that long caches still fill the GPU;
// each split produces a normalised partial output and its log-sum-exp, and a
// second kernel merges them (FlashAttention-3 page, split-K combine).
//
// The G = Hq / Hkv query heads that share a key/value head are the rows of one
// 128-row query tile, so each split is a small attention problem: S = Q K^T over
// 128-key tiles with tcgen05.mma into TMEM (double buffered: S(j+1) is computed
// while the softmax works on S(j)), an online softmax per row on the CUDA cores,
// and O += P V with P from TMEM. The tensor core does the per-element work of
// reading K and V from shared memory, so a block streams at the rate TMA and
// HBM deliver rather than at the CUDA cores' instruction rate. Rows past G
// (other heads, or zeros) ride along in the MMAs; their results are discarded.
// 224 threads:
//   warps 0-3   stage the query rows into the swizzled operand layout (zeros
//               past the group's heads), then softmax and epilogue, warp w for
//               rows 32w .. 32w+31 (its TMEM lane quadrant); only the first
//               ceil(rows/32) warps take part in those;
//   warp 4      MMA issuer: S(0), S(1), PV(0), S(2), PV(1), ...;
//   warps 5, 6  TMA producers: K and V tiles of the split into a ring of
//               shared-memory slots, in the order the MMAs consume them
//               (K_0 K_1 V_0 K_2 V_1 ...); boxes split between the two threads.
// TMEM columns: S buffers [0, 128) and [128, 256), O [256, 256 + D).
#pragma once

#include "sm100_ptx.cuh"

namespace eab {

struct DecodeParams {
    const void* q;           // [B, Hq, D], the input type
    float* o_part;           // [B, Hq, S, D]
    float* lse_part;         // [B, Hq, S]
    int B, Hq, Hkv, L, S, chunk;  // chunk: keys per split, a multiple of 128
    int G, groups;                // G = Hq / Hkv; groups of 128 query heads per KV head
    float scale_log2;
};

template <int D>
struct DecCfg {
    static constexpr int BM = 128;  // query rows per tile (heads of one KV head)
    static constexpr int BN = 128;  // keys per tile
    static constexpr int CHUNKS = D / 64;
    static constexpr int Q_BYTES = BM * D * 2;
    static constexpr int TILE_BYTES = BN * D * 2;
    static constexpr int SLOTS = (D == 128) ? 6 : 12;
    static constexpr int NUM_THREADS = 224;
    // q_ready, slot_full, slot_empty, s_full[2], p_full[2], o_done[2], drain
    static constexpr int NUM_BARRIERS = 1 + 2 * SLOTS + 2 + 2 + 2 + 1;
    static constexpr int SMEM_BYTES = 1024 + Q_BYTES + SLOTS * TILE_BYTES + NUM_BARRIERS * 8 + 16;
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr float RESCALE_THRESHOLD = 8.0f;  // log2 units
};

// Position of K_j / V_j in the split's load order (the MMA's consumption order)
// K_0 K_1 V_0 K_2 V_1 ... K_{n-1} V_{n-2} V_{n-1}; dec_load_kind inverts it.
__device__ __forceinline__ int dec_kpos(int j) { return j == 0 ? 0 : 2 * j - 1; }
__device__ __forceinline__ int dec_vpos(int j, int n) { return j == n - 1 ? 2 * n - 1 : 2 * j + 2; }
__device__ __forceinline__ bool dec_load_kind(int i, int n, int* j) {
    if (i == 2 * n - 1) { *j = n - 1; return true; }
    if (i == 0) { *j = 0; return false; }
    if (i & 1) { *j = (i + 1) >> 1; return false; }
    *j = (i >> 1) - 1;
    return true;
}

template <int D, class E>
__global__ void __launch_bounds__(224, 1)
    decode_splitkv_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                     const DecodeParams p) {
    using C = DecCfg<D>;
    constexpr int BM = C::BM, BN = C::BN, SLOTS = C::SLOTS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = smem;
    uint8_t* sKV = smem + C::Q_BYTES;
    uint64_t* bars = reinterpret_cast<uint64_t*>(sKV + SLOTS * C::TILE_BYTES);
    uint64_t* q_ready = bars;                  // query rows staged (one arrival per warp 0-3)
    uint64_t* slot_full = q_ready + 1;         // [SLOTS]
    uint64_t* slot_empty = slot_full + SLOTS;  // [SLOTS]
    uint64_t* s_full = slot_empty + SLOTS;     // [2]
    uint64_t* p_full = s_full + 2;             // [2] (one arrival per softmax warp)
    // P V(j) completes phase j >> 1 of o_done[j & 1]. One barrier per parity:
    // S(j) done implies only P V(j-2) done, so a single barrier could be two
    // phases behind a waiter and its parity test would pass too early.
    uint64_t* o_done = p_full + 2;
    uint64_t* drain = o_done + 2;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int split = blockIdx.x;
    const int hk = blockIdx.y / p.groups, grp = blockIdx.y % p.groups;
    const int b = blockIdx.z;
    const int h0 = hk * p.G + grp * BM;              // first query head of this tile
    const int rows = min(BM, p.G - grp * BM);        // real query rows
    const int nsw = (rows + 31) / 32;                // softmax warps taking part
    const int k0 = split * p.chunk;
    const int k1 = min(p.L, k0 + p.chunk);
    const int nt = k1 > k0 ? (k1 - k0 + BN - 1) / BN : 0;

    if (threadIdx.x == 0) {
        mbar_init(q_ready, 4);
        for (int i = 0; i < SLOTS; ++i) {
            mbar_init(&slot_full[i], C::CHUNKS);
            mbar_init(&slot_empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s_full[i], 1);
            mbar_init(&p_full[i], nsw);
        }
        mbar_init(&o_done[0], 1);
        mbar_init(&o_done[1], 1);
        mbar_init(drain, 1);
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
    grid_dep_wait();  // the previous kernel's writes are visible from here on

    if (warp >= 5) {
        // ------------------------------------------------------ producers ---
        if (lane == 0 && nt > 0) {
            const int me = warp - 5;
            constexpr uint32_t BOX_BYTES = BN * 128;
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            const int z = b * p.Hkv + hk;
            int issued = 0;
            for (int i = 0; i < 2 * nt; ++i) {
                bool mine = false;
#pragma unroll
                for (int c = 0; c < C::CHUNKS; ++c) mine |= ((i * C::CHUNKS + c) & 1) == me;
                if (!mine) continue;
                const int slot = i % SLOTS, use = i / SLOTS;
                if (use > 0 && !mbar_wait(&slot_empty[slot], (use - 1) & 1, abort_flag)) break;
                int j;
                const CUtensorMap* tm = dec_load_kind(i, nt, &j) ? &tm_v : &tm_k;
                uint8_t* dst = sKV + slot * C::TILE_BYTES;
#pragma unroll
                for (int c = 0; c < C::CHUNKS; ++c) {
                    if (((i * C::CHUNKS + c) & 1) != me) continue;
                    mbar_arrive_expect_tx(&slot_full[slot], BOX_BYTES);
                    tma_load_3d(dst + c * BOX_BYTES, tm, &slot_full[slot], c * 64, k0 + j * BN, z);
                }
                issued = i + 1;
            }
            // Every load of this CTA is issued: the next kernel in the stream may be
            // scheduled (it waits for this grid's completion before reading memory).
            grid_dep_launch();
            // Let every copy in flight land before the CTA can exit.
            for (int i = max(0, issued - SLOTS); i < issued; ++i)
                mbar_wait(&slot_full[i % SLOTS], (i / SLOTS) & 1, nullptr);
        }
    } else if (warp == 4) {
        // ---------------------------------------------------- MMA issuer ----
        if (lane == 0 && nt > 0) {
            constexpr uint32_t idesc_qk = make_idesc(BM, BN, 0, 0, E::fmt);
            constexpr uint32_t idesc_pv = make_idesc(BM, D, 0, 1, E::fmt);
            const uint32_t o_tmem = tmem + 256;
            const uint32_t q_addr = smem_addr(sQ), kv_addr = smem_addr(sKV);
            bool ok = mbar_wait(q_ready, 0, abort_flag);
            auto issue_s = [&](int j) -> bool {
                const int ik = dec_kpos(j);
                if (!mbar_wait(&slot_full[ik % SLOTS], (ik / SLOTS) & 1, abort_flag)) return false;
                tc_fence_after();
                const uint32_t k_addr = kv_addr + (ik % SLOTS) * C::TILE_BYTES;
                const uint32_t s_tmem = tmem + (j & 1) * 128;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t koff = (kk & 3) * 32;
                    const uint64_t ad = make_sdesc_sw128(q_addr + (kk >> 2) * (BM * 128) + koff, 16, 1024);
                    const uint64_t bd = make_sdesc_sw128(k_addr + (kk >> 2) * (BN * 128) + koff, 16, 1024);
                    mma_ss(s_tmem, ad, bd, idesc_qk, kk > 0 ? 1u : 0u);
                }
                tc_commit(&s_full[j & 1]);
                tc_commit(&slot_empty[ik % SLOTS]);
                return true;
            };
            if (ok) ok = issue_s(0);
            if (ok && nt > 1) ok = issue_s(1);
            for (int j = 0; ok && j < nt; ++j) {
                // O += P(j) V_j, then S(j+2) into the S buffer this product reads
                const int iv = dec_vpos(j, nt);
                ok = mbar_wait(&slot_full[iv % SLOTS], (iv / SLOTS) & 1, abort_flag) &&
                     mbar_wait_spin(&p_full[j & 1], (j >> 1) & 1, abort_flag);
                if (!ok) break;
                tc_fence_after();
                const uint32_t v_addr = kv_addr + (iv % SLOTS) * C::TILE_BYTES;
                const uint32_t p_tmem = tmem + (j & 1) * 128;
#pragma unroll
                for (int kk = 0; kk < BN / 16; ++kk) {
                    const uint64_t bd = make_sdesc_sw128(v_addr + kk * 16 * 128, BN * 128, 1024);
                    mma_ts(o_tmem, p_tmem + kk * 8, bd, idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
                }
                tc_commit(&o_done[j & 1]);
                tc_commit(&slot_empty[iv % SLOTS]);
                if (j + 2 < nt) ok = issue_s(j + 2);
            }
            // Every MMA must be complete before TMEM is released.
            tc_commit(drain);
            mbar_wait(drain, 0, nullptr);
        }
        __syncwarp();
    } else {
        // ------------------------------------------- query staging, softmax ----
        const int row = warp * 32 + lane;
        const bool real = row < rows;
        const size_t out_row = static_cast<size_t>(b) * p.Hq + h0 + row;
        if (nt > 0) {
            // this warp's 32 query rows in the K-major 128-byte-swizzled operand
            // layout (rows past the group's heads as zeros)
#pragma unroll
            for (int c = 0; c < D / 8; ++c) {
                uint4 v4 = make_uint4(0u, 0u, 0u, 0u);
                if (real) v4 = *reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p.q) + out_row * D + c * 8);
                *reinterpret_cast<uint4*>(sQ + (c >> 3) * (BM * 128) + row * 128 + (((c & 7) ^ (row & 7)) << 4)) = v4;
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(q_ready);
        }
        if (warp >= nsw) {
            // no real rows in this quadrant
        } else if (nt == 0) {
            // an empty split: weight 0 in the combine
            if (real) {
                p.lse_part[out_row * p.S + split] = -INFINITY;
#pragma unroll 4
                for (int c = 0; c < D; c += 4)
                    *reinterpret_cast<float4*>(p.o_part + (out_row * p.S + split) * D + c) = make_float4(0.f, 0.f, 0.f, 0.f);
            }
        } else {
            const uint32_t lane_base = tmem + (uint32_t(warp * 32) << 16);
            const uint32_t o_addr = lane_base + 256;
            const float c2 = p.scale_log2;
            float m_used = -INFINITY, l = 0.f;
            bool ok = true;
            for (int j = 0; j < nt; ++j) {
                const uint32_t s_addr = lane_base + (j & 1) * 128;
                const bool w1 = mbar_wait(&s_full[j & 1], (j >> 1) & 1, abort_flag);
                if (!__all_sync(0xffffffffu, w1)) { ok = false; break; }
                tc_fence_after();
                const int lim = min(BN, k1 - (k0 + j * BN));  // valid keys of this tile
                float mx = -INFINITY;
                uint32_t sv[128];
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    tmem_ld64(s_addr + h * 64, reinterpret_cast<uint32_t(&)[64]>(sv[h * 64]));
                }
                if (lim < BN) {
#pragma unroll
                    for (int i = 0; i < 128; ++i)
                        if (i >= lim) sv[i] = 0xff800000u;  // -inf: exp2 gives 0
                }
#pragma unroll
                for (int i = 0; i < 128; i += 2) mx = max3(mx, __uint_as_float(sv[i]), __uint_as_float(sv[i + 1]));
                const float m_tile = mx * c2;
                const bool need = m_tile > m_used + C::RESCALE_THRESHOLD;
                float factor = 1.f;
                if (need) {
                    factor = ex2_approx(m_used - m_tile);
                    m_used = m_tile;
                }
                l *= factor;
                if (j > 0 && __any_sync(0xffffffffu, need)) {
                    // O must hold P V(j-1) before it is rescaled (S(j) implies only P V(j-2))
                    const bool w3 = mbar_wait(&o_done[(j - 1) & 1], ((j - 1) >> 1) & 1, abort_flag);
                    if (!__all_sync(0xffffffffu, w3)) { ok = false; break; }
                    tc_fence_after();
#pragma unroll
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t r3[32];
                        tmem_ld32(o_addr + c * 32, r3);
#pragma unroll
                        for (int i = 0; i < 32; ++i) r3[i] = __float_as_uint(__uint_as_float(r3[i]) * factor);
                        tmem_st32(o_addr + c * 32, r3);
                    }
                }
                const float2 c2x2 = make_float2(c2, c2), negm2 = make_float2(-m_used, -m_used);
                float2 rsum[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) rsum[k] = make_float2(0.f, 0.f);
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    uint32_t pk[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const int e = h * 64 + 2 * i;
                        const float2 y = ffma2(make_float2(__uint_as_float(sv[e]), __uint_as_float(sv[e + 1])), c2x2, negm2);
                        const float2 pp = make_float2(ex2_approx(y.x), ex2_approx(y.y));
                        rsum[i & 3] = fadd2(rsum[i & 3], pp);
                        pk[i] = E::pack2(pp.x, pp.y);
                    }
                    tmem_st32(s_addr + h * 32, pk);
                }
                const float2 rs = fadd2(fadd2(rsum[0], rsum[1]), fadd2(rsum[2], rsum[3]));
                l += rs.x + rs.y;
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&p_full[j & 1]);
            }
            if (ok && __all_sync(0xffffffffu, mbar_wait(&o_done[(nt - 1) & 1], ((nt - 1) >> 1) & 1, abort_flag))) {
                tc_fence_after();
                const float inv_l = 1.f / l;
                float* dst = p.o_part + (out_row * p.S + split) * D;
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t r3[32];
                    tmem_ld32(o_addr + c * 32, r3);
                    if (real) {
#pragma unroll
                        for (int i = 0; i < 32; i += 4)
                            *reinterpret_cast<float4*>(dst + c * 32 + i) =
                                make_float4(__uint_as_float(r3[i]) * inv_l, __uint_as_float(r3[i + 1]) * inv_l,
                                            __uint_as_float(r3[i + 2]) * inv_l, __uint_as_float(r3[i + 3]) * inv_l);
                    }
                }
                if (real) p.lse_part[out_row * p.S + split] = (m_used + log2f(l)) * 0.69314718055994530942f;
            } else if (real) {
                // a wait was abandoned (timeout, recorded in the status word): leave an
                // empty partial (zero weight in the combine) rather than stale memory
                float* dst = p.o_part + (out_row * p.S + split) * D;
                for (int c = 0; c < D; c += 4) *reinterpret_cast<float4*>(dst + c) = make_float4(0.f, 0.f, 0.f, 0.f);
                p.lse_part[out_row * p.S + split] = -INFINITY;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 4) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

// ---------------------------------------------- decode, keys as tile rows ----
// The same split-KV partials for a small group (G = Hq / Hkv <= 32 query heads
// per key/value head, d = 128), computed transposed so that the 128 keys of a
// tile, not the few query heads, fill the 128 rows of the tensor-core tile:
//   S^T = K_j Q^T    tcgen05.mma, A = K_j (128 keys x d, K-major, as TMA lands
//                    it), B = the group's queries (NQ = 16 or 32 rows, zeros past
//                    G) -> TMEM, 128 lanes (keys) x NQ columns;
//   softmax          thread t owns key t of the tile: its NQ scores, per query
//                    column a maximum over the 128 keys (warp shuffles, then the
//                    four warps through shared memory), the lazy rescale
//                    (threshold 2^8, log2 units), NQ exponentials per thread
//                    instead of 128, a per-thread partial sum of p per column;
//                    P (bf16) goes to shared memory as a K-major operand;
//   O^T += V_j^T P   tcgen05.mma, A = V_j read MN-major (the head dimension is
//                    contiguous), B = P -> TMEM, 128 lanes (head dim) x NQ.
// The exp2 work per tile drops from 128 x 128 to 128 x NQ, so a block streams
// K and V at the rate TMA and HBM deliver, and TMEM use drops to 64 or 128
// columns. Warp roles and the K_0 K_1 V_0 K_2 V_1 ... load order are those of
// decode_splitkv_kernel. TMEM columns: S^T buffers [0, NQ), [NQ, 2 NQ), O^T
// [2 NQ, 3 NQ).
template <int NQ, int SLOTS_ = 6>
struct DecTCfg {
    static constexpr int D = 128, BN = 128, CHUNKS = D / 64;
    static constexpr int Q_BYTES = CHUNKS * NQ * 128;  // queries as the B operand, [chunk][NQ rows][128 B]
    static constexpr int P_BYTES = 2 * NQ * 128;       // P as the B operand, [key chunk][NQ rows][128 B]
    static constexpr int TILE_BYTES = BN * D * 2;
    static constexpr int SLOTS = SLOTS_;
    static constexpr int NUM_THREADS = 224;
    static constexpr int BLOCKS_PER_SM = SLOTS <= 3 ? 2 : 1;  // shared memory: 6 slots take a whole SM
    static constexpr int RED_FLOATS = 3 * 4 * NQ;      // column maxima (two buffers) and sums of the four warps
    // q_ready, slot_full, slot_empty, s_full[2], p_full[2], o_done[2], drain, red_bar[2], sum_bar
    static constexpr int NUM_BARRIERS = 1 + 2 * SLOTS + 2 + 2 + 2 + 1 + 2 + 1;
    static constexpr int SMEM_BYTES =
        1024 + Q_BYTES + 2 * P_BYTES + SLOTS * TILE_BYTES + RED_FLOATS * 4 + NUM_BARRIERS * 8 + 16;
    static constexpr uint32_t TMEM_COLS = NQ <= 16 ? 64 : 128;
    static constexpr float RESCALE_THRESHOLD = 8.0f;
};

template <int NQ>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&r)[NQ]) {
    if constexpr (NQ == 16) tmem_ld16(taddr, r);
    else tmem_ld32(taddr, r);
}
template <int NQ>
__device__ __forceinline__ void tmem_st_cols(uint32_t taddr, const uint32_t (&r)[NQ]) {
    if constexpr (NQ == 16) tmem_st16(taddr, r);
    else tmem_st32(taddr, r);
}

template <int NQ, int SLOTS_, class E>
__global__ void __launch_bounds__(224, DecTCfg<NQ, SLOTS_>::BLOCKS_PER_SM)
    decode_splitkv_keys_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                               const DecodeParams p) {
    using C = DecTCfg<NQ, SLOTS_>;
    constexpr int D = C::D, BN = C::BN, SLOTS = C::SLOTS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = smem;
    uint8_t* sP = sQ + C::Q_BYTES;                 // two P buffers
    uint8_t* sKV = sP + 2 * C::P_BYTES;
    float* red = reinterpret_cast<float*>(sKV + SLOTS * C::TILE_BYTES);  // [3][4][NQ]
    uint64_t* bars = reinterpret_cast<uint64_t*>(red + C::RED_FLOATS);
    uint64_t* q_ready = bars;                  // queries staged (one arrival per warp 0-3)
    uint64_t* slot_full = q_ready + 1;         // [SLOTS]
    uint64_t* slot_empty = slot_full + SLOTS;  // [SLOTS]
    uint64_t* s_full = slot_empty + SLOTS;     // [2]
    uint64_t* p_full = s_full + 2;             // [2] (one arrival per softmax warp)
    uint64_t* o_done = p_full + 2;             // [2] P V(j) completes phase j >> 1 of o_done[j & 1]
    uint64_t* drain = o_done + 2;
    uint64_t* red_bar = drain + 1;             // [2] the four softmax warps' column maxima of a tile
    uint64_t* sum_bar = red_bar + 2;           // the four softmax warps' column sums
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sum_bar + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int split = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
    const int G = p.G;                                    // query heads of this group (<= NQ)
    const size_t row0 = static_cast<size_t>(b) * p.Hq + static_cast<size_t>(hk) * G;  // first output row
    const int k0 = split * p.chunk;
    const int k1 = min(p.L, k0 + p.chunk);
    const int nt = k1 > k0 ? (k1 - k0 + BN - 1) / BN : 0;

    if (threadIdx.x == 0) {
        mbar_init(q_ready, 4);
        for (int i = 0; i < SLOTS; ++i) {
            mbar_init(&slot_full[i], C::CHUNKS);
            mbar_init(&slot_empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s_full[i], 1);
            mbar_init(&p_full[i], 4);
            mbar_init(&o_done[i], 1);
        }
        mbar_init(drain, 1);
        mbar_init(&red_bar[0], 4);
        mbar_init(&red_bar[1], 4);
        mbar_init(sum_bar, 4);
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
    grid_dep_wait();  // the previous kernel's writes are visible from here on

    if (warp >= 5) {
        // ------------------------------------------------------ producers ---
        if (lane == 0 && nt > 0) {
            const int me = warp - 5;
            constexpr uint32_t BOX_BYTES = BN * 128;
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            const int z = b * p.Hkv + hk;
            int issued = 0;
            for (int i = 0; i < 2 * nt; ++i) {
                bool mine = false;
#pragma unroll
                for (int c = 0; c < C::CHUNKS; ++c) mine |= ((i * C::CHUNKS + c) & 1) == me;
                if (!mine) continue;
                const int slot = i % SLOTS, use = i / SLOTS;
                if (use > 0 && !mbar_wait(&slot_empty[slot], (use - 1) & 1, abort_flag)) break;
                int j;
                const CUtensorMap* tm = dec_load_kind(i, nt, &j) ? &tm_v : &tm_k;
                uint8_t* dst = sKV + slot * C::TILE_BYTES;
#pragma unroll
                for (int c = 0; c < C::CHUNKS; ++c) {
                    if (((i * C::CHUNKS + c) & 1) != me) continue;
                    mbar_arrive_expect_tx(&slot_full[slot], BOX_BYTES);
                    tma_load_3d(dst + c * BOX_BYTES, tm, &slot_full[slot], c * 64, k0 + j * BN, z);
                }
                issued = i + 1;
            }
            // Every load of this CTA is issued: the next kernel in the stream may be
            // scheduled (it waits for this grid's completion before reading memory).
            grid_dep_launch();
            // Let every copy in flight land before the CTA can exit.
            for (int i = max(0, issued - SLOTS); i < issued; ++i)
                mbar_wait(&slot_full[i % SLOTS], (i / SLOTS) & 1, nullptr);
        }
    } else if (warp == 4) {
        // ---------------------------------------------------- MMA issuer ----
        if (lane == 0 && nt > 0) {
            constexpr uint32_t idesc_s = make_idesc(BN, NQ, 0, 0, E::fmt);  // M = keys, N = queries
            constexpr uint32_t idesc_o = make_idesc(D, NQ, 1, 0, E::fmt);   // M = head dim (V read MN-major)
            const uint32_t o_tmem = tmem + 2 * NQ;
            const uint32_t q_addr = smem_addr(sQ), p_addr = smem_addr(sP), kv_addr = smem_addr(sKV);
            bool ok = mbar_wait(q_ready, 0, abort_flag);
            auto issue_s = [&](int j) -> bool {
                const int ik = dec_kpos(j);
                if (!mbar_wait(&slot_full[ik % SLOTS], (ik / SLOTS) & 1, abort_flag)) return false;
                tc_fence_after();
                const uint32_t k_addr = kv_addr + (ik % SLOTS) * C::TILE_BYTES;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t koff = (kk & 3) * 32;
                    const uint64_t ad = make_sdesc_sw128(k_addr + (kk >> 2) * (BN * 128) + koff, 16, 1024);
                    const uint64_t bd = make_sdesc_sw128(q_addr + (kk >> 2) * (NQ * 128) + koff, 16, 1024);
                    mma_ss(tmem + (j & 1) * NQ, ad, bd, idesc_s, kk > 0 ? 1u : 0u);
                }
                tc_commit(&s_full[j & 1]);
                tc_commit(&slot_empty[ik % SLOTS]);
                return true;
            };
            if (ok) ok = issue_s(0);
            if (ok && nt > 1) ok = issue_s(1);
            for (int j = 0; ok && j < nt; ++j) {
                // O^T += V_j^T P(j), then S^T(j+2) into the S buffer P(j) came from
                const int iv = dec_vpos(j, nt);
                ok = mbar_wait(&slot_full[iv % SLOTS], (iv / SLOTS) & 1, abort_flag) &&
                     mbar_wait_spin(&p_full[j & 1], (j >> 1) & 1, abort_flag);
                if (!ok) break;
                tc_fence_after();
                const uint32_t v_addr = kv_addr + (iv % SLOTS) * C::TILE_BYTES;
                const uint32_t pb = p_addr + (j & 1) * C::P_BYTES;
#pragma unroll
                for (int kk = 0; kk < BN / 16; ++kk) {
                    // 16 keys per step: rows kk*16.. of the V tile (MN-major A, the
                    // head dimension's two 64-column chunks BN * 128 bytes apart), and
                    // 32 bytes of every P row (K-major B)
                    const uint64_t ad = make_sdesc_sw128(v_addr + kk * 16 * 128, BN * 128, 1024);
                    const uint64_t bd = make_sdesc_sw128(pb + (kk >> 2) * (NQ * 128) + (kk & 3) * 32, 16, 1024);
                    mma_ss(o_tmem, ad, bd, idesc_o, (j > 0 || kk > 0) ? 1u : 0u);
                }
                tc_commit(&o_done[j & 1]);
                tc_commit(&slot_empty[iv % SLOTS]);
                if (j + 2 < nt) ok = issue_s(j + 2);
            }
            // Every MMA must be complete before TMEM is released.
            tc_commit(drain);
            mbar_wait(drain, 0, nullptr);
        }
        __syncwarp();
    } else {
        // ------------------------------------------- query staging, softmax ----
        const int t = threadIdx.x;  // key t of each tile; lane t of S^T and of O^T (head-dim element t)
        if (nt > 0) {
            // the group's queries as NQ rows of the K-major 128-byte-swizzled operand
            // (rows past G as zeros): 16-byte unit u of row r of chunk c sits at
            // unit u ^ (r & 7)
            for (int i = t; i < NQ * (D / 8); i += 128) {
                const int r = i / (D / 8), u = i % (D / 8);
                uint4 v4 = make_uint4(0u, 0u, 0u, 0u);
                if (r < G) v4 = *reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p.q) + (row0 + r) * D + u * 8);
                *reinterpret_cast<uint4*>(sQ + (u >> 3) * (NQ * 128) + r * 128 + (((u & 7) ^ (r & 7)) << 4)) = v4;
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(q_ready);
        }
        if (nt == 0) {
            // an empty split: weight 0 in the combine
            for (int c = 0; c < G; ++c) p.o_part[((row0 + c) * p.S + split) * D + t] = 0.f;
            if (t < G) p.lse_part[(row0 + t) * p.S + split] = -INFINITY;
        } else {
            const uint32_t lane_base = tmem + (uint32_t(warp * 32) << 16);
            const uint32_t o_addr = lane_base + 2 * NQ;
            const float c2 = p.scale_log2;
            float m_used[NQ], lsum[NQ];
#pragma unroll
            for (int c = 0; c < NQ; ++c) {
                m_used[c] = -INFINITY;
                lsum[c] = 0.f;
            }
            bool ok = true;
            for (int j = 0; j < nt; ++j) {
                const bool w1 = mbar_wait(&s_full[j & 1], (j >> 1) & 1, abort_flag);
                if (!__all_sync(0xffffffffu, w1)) { ok = false; break; }
                tc_fence_after();
                uint32_t sv[NQ];
                tmem_ld_cols<NQ>(lane_base + (j & 1) * NQ, sv);
                const bool valid = k0 + j * BN + t < k1;
                float s2[NQ];
#pragma unroll
                for (int c = 0; c < NQ; ++c) s2[c] = valid ? __uint_as_float(sv[c]) * c2 : -INFINITY;
                // per query column: maximum over the tile's 128 keys
                float* rmax = red + (j & 1) * 4 * NQ;
#pragma unroll
                for (int c = 0; c < NQ; ++c) {
                    if (c < G) {
                        float m = s2[c];
#pragma unroll
                        for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
                        if (lane == 0) rmax[warp * NQ + c] = m;
                    }
                }
                // exchange through an mbarrier (a bounded wait: no warp can hang the
                // others if one gives up); tile j completes phase j >> 1 of
                // red_bar[j & 1], and no warp arrives for tile j + 2 before every warp
                // has passed tile j + 1
                __syncwarp();
                if (lane == 0) mbar_arrive(&red_bar[j & 1]);
                const bool w2 = mbar_wait(&red_bar[j & 1], (j >> 1) & 1, abort_flag);
                if (!__all_sync(0xffffffffu, w2)) { ok = false; break; }
                bool any = false;
                float factor[NQ];
#pragma unroll
                for (int c = 0; c < NQ; ++c) {
                    factor[c] = 1.f;
                    if (c < G) {
                        const float mt = fmaxf(fmaxf(rmax[c], rmax[NQ + c]), fmaxf(rmax[2 * NQ + c], rmax[3 * NQ + c]));
                        if (mt > m_used[c] + C::RESCALE_THRESHOLD) {
                            factor[c] = ex2_approx(m_used[c] - mt);
                            m_used[c] = mt;
                            any = true;
                        }
                    }
                    lsum[c] *= factor[c];
                }
                // every thread of the four warps takes the same decision (the maxima are shared)
                if (j > 0 && any) {
                    // O^T must hold P V(j-1) before it is rescaled (S(j) implies only P V(j-2))
                    const bool w3 = mbar_wait(&o_done[(j - 1) & 1], ((j - 1) >> 1) & 1, abort_flag);
                    if (!__all_sync(0xffffffffu, w3)) { ok = false; break; }
                    tc_fence_after();
                    uint32_t ov[NQ];
                    tmem_ld_cols<NQ>(o_addr, ov);
#pragma unroll
                    for (int c = 0; c < NQ; ++c) ov[c] = __float_as_uint(__uint_as_float(ov[c]) * factor[c]);
                    tmem_st_cols<NQ>(o_addr, ov);
                    tmem_st_wait();
                }
                // P(j): p = exp2(s * c2 - m) for the real columns, into the P buffer
                // of this parity (P V(j-2), its last reader, is complete: S(j) is)
                uint8_t* pb = sP + (j & 1) * C::P_BYTES + (t >> 6) * (NQ * 128) + (t & 7) * 2;
                const int unit = (t & 63) >> 3;
#pragma unroll
                for (int c = 0; c < NQ; ++c) {
                    float pv = 0.f;
                    if (c < G) {
                        pv = ex2_approx(s2[c] - m_used[c]);
                        lsum[c] += pv;
                    }
                    *reinterpret_cast<typename E::T*>(pb + c * 128 + ((unit ^ (c & 7)) << 4)) = E::from_float(pv);
                }
                fence_proxy_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&p_full[j & 1]);
            }
            // l per column: the sum of the 128 threads' partial sums
            float* rsum = red + 2 * 4 * NQ;
            if (ok) {
#pragma unroll
                for (int c = 0; c < NQ; ++c) {
                    if (c < G) {
                        float sm = lsum[c];
#pragma unroll
                        for (int off = 16; off > 0; off >>= 1) sm += __shfl_xor_sync(0xffffffffu, sm, off);
                        if (lane == 0) rsum[warp * NQ + c] = sm;
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(sum_bar);
            ok = ok && __all_sync(0xffffffffu, mbar_wait(sum_bar, 0, abort_flag));
            ok = ok && __all_sync(0xffffffffu, mbar_wait(&o_done[(nt - 1) & 1], ((nt - 1) >> 1) & 1, abort_flag));
            if (ok) {
                tc_fence_after();
                uint32_t ov[NQ];
                tmem_ld_cols<NQ>(o_addr, ov);
#pragma unroll
                for (int c = 0; c < NQ; ++c) {
                    if (c < G) {
                        const float l = (rsum[c] + rsum[NQ + c]) + (rsum[2 * NQ + c] + rsum[3 * NQ + c]);
                        p.o_part[((row0 + c) * p.S + split) * D + t] = __uint_as_float(ov[c]) / l;
                        if (t == c) p.lse_part[(row0 + c) * p.S + split] = (m_used[c] + log2f(l)) * 0.69314718055994530942f;
                    }
                }
            } else {
                // a wait was abandoned (timeout, recorded in the status word): leave
                // empty partials (zero weight in the combine) rather than stale memory
                for (int c = 0; c < G; ++c) p.o_part[((row0 + c) * p.S + split) * D + t] = 0.f;
                if (t < G) p.lse_part[(row0 + t) * p.S + split] = -INFINITY;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 4) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

// ------------------------------------------------------------- combine ------
// One block per (b, h), D threads: M = max_s lse_s, w_s = exp(lse_s - M),
// O = sum_s w_s O_s / sum_s w_s, LSE = M + ln(sum_s w_s).
template <int D, class E>
__global__ void __launch_bounds__(D)
    combine_kernel(const float* __restrict__ o_part, const float* __restrict__ lse_part,
                   typename E::T* __restrict__ o, float* __restrict__ lse, int S) {
    extern __shared__ float w_s[];  // S weights
    __shared__ float red[D / 32];
    __shared__ float bcast;
    const int bh = blockIdx.x, t = threadIdx.x;
    grid_dep_wait();  // the partials of the decode before it are complete and visible
    grid_dep_launch();
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
    o[static_cast<size_t>(bh) * D + t] = E::from_float(none ? 0.f : acc / wsum);
    if (t == 0) lse[bh] = none ? -INFINITY : M + logf(wsum);
}

}  // namespace eab
