// Prefill forward pass on sm_100a: O = softmax(scale * Q K^T) V and the per-row
// log-sum-exp.
//
// The method is the tiled online softmax of "1-Flash-Attention.md" (sections
// "Tiling（分块）技术", "递归计算softmax"): a query tile stays on chip while key /
// value tiles stream past it; per row a running max m and denominator l are
// kept, the accumulator is rescaled when the max moves, and O is divided by l
// once at the end (FlashAttention V2 page: fewer non-matmul operations). Loop
// order is the V2 one (query tiles outer, key/value tiles inner), and work is
// spread over thread blocks by sequence position as well as by head.
//
// B200 mapping. A persistent grid (one CTA per SM) walks a list of work items;
// an item is one 256-row query block of one (batch, head), processed as two
// 128-row query tiles that share every K/V tile. Causal items are ordered
// heaviest first and dealt to the CTAs in snake order; non-causal items head by
// head, so that the query blocks of one head run in the same wave and share its
// K/V tiles through L2, and a CTA takes its first item by its index and each
// later one from a per-launch counter (the first producer thread takes it and
// hands it to the other roles through a small ring in shared memory), so the
// CTAs finish together. A non-causal problem whose last round would hold at most
// half as many query blocks as there are SMs runs that round as a second launch
// (the SPLIT kernel) in 128-row halves: the two query tiles of a CTA take the same
// rows against the first and the second half of the key tiles (each K/V tile
// then serves one tile only), and tile 1 merges the two partial results as the
// online softmax merges two blocks of keys. 384 threads,
// warp-specialised:
//   warps 0-3   softmax of query tile 0, one thread per row (TMEM lane), and
//               its epilogue: O/l rounded to the input type, staged per warp in
//               shared memory as a 128-byte-swizzled 32-row box and written by
//               one bulk tensor store per 64 columns (the F32OUT kernels keep O
//               in fp32, read the staging back and store whole 128-byte row
//               segments);
//   warps 4-7   the same for query tile 1;
//   warp 8, 9   MMA issuers, one per query tile. A thread that has just issued
//               tcgen05.mma cannot act on an mbarrier for several hundred cycles,
//               so two issuing warps keep the tensor core busy while each waits;
//   warps 10,11 TMA producers: the Q tiles of each item, then K_j and V_j into a
//               ring of shared-memory slots (full/empty mbarriers). One issuing
//               thread streams TMA boxes one after another, so the boxes of
//               every tile are split between two threads. They run key tiles
//               ahead and wait with suspended try_wait, taking no issue slots
//               from the softmax warps of their sub-partitions.
// Per query tile t and key tile j:
//   S_t = Q_t K_j^T           tcgen05.mma (A, B K-major in smem) -> TMEM S_t;
//   softmax                   pass 1 reads S_t and takes the row max; when it has
//                             grown by more than 2^8 (log2 units) O_t is rescaled
//                             in TMEM (lazy rescale); the two softmax warpgroups
//                             then take turns for pass 2, which computes
//                             p = exp2(s*scale*log2e - m) with one FMA, sums l in
//                             fp32 and writes P_t in the input type (bf16 or
//                             fp16, the E template parameter) over the S_t columns,
//                             announcing each half (64 keys) as it lands;
//   O_t += P_t V_j            tcgen05.mma with A = P_t from TMEM, B = V_j MN-major,
//                             the first 64 keys while the softmax still works on
//                             the second 64. The issuer waits on P by polling
//                             (a suspended wait resumes late).
// S_t(j+1) is issued after O_t += P_t(j) V_j by the same thread, so the tensor
// pipe's issue order keeps P_t(j) intact until it has been read, and S_t(j+1)'s
// completion implies that O_t holds every earlier P V product. Between items
// the next Q tile is loaded as soon as the last S MMA of its buffer completes,
// and the next item's first P V waits only until the epilogue has read O_t.
// Every barrier phase is counted across items.
// TMEM columns: tile t uses S [256t, 256t+128) and O [256t+128, 256t+128+D).
#pragma once

#include "sm100_ptx.cuh"

namespace eab {

struct FwdParams {
    void* o;           // [B, Hq, N, D]: the input type (bf16 / fp16), or fp32 for F32OUT
    float* lse;        // [B, Hq, N]
    int B, Hq, Hkv, N;
    int n_qblocks;     // ceil(N / 256)
    int n_items;       // work items of this launch
    int block0;        // split launches: the first query block; item w is half w & 1 of block block0 + w / 2
    int chained;       // split launches: 1 when the launch of the call's other blocks precedes this one
    float scale_log2;  // scale * log2(e)
    int sched_slot;    // this launch's work counter in g_fwd_sched
};

// Dynamic work distribution (non-causal launches): a CTA takes its first item by
// its index and every later one from a counter, in the list's order, so the
// CTAs finish together whatever each item actually costs. Each launch uses its
// own counter slot (the host cycles through them); the last CTA to finish resets
// the slot to zero for its next use. Causal launches deal their items statically
// (fwd_work_index): with items from 31 down to 3 key-tile units, heaviest first,
// the static snake order already reaches the makespan of a greedy longest-first
// schedule and saves the counter's hand-over at every item.
constexpr int kFwdSchedSlots = 64;
__device__ unsigned int g_fwd_sched[kFwdSchedSlots][2];  // [items taken past the first round, CTAs done]

template <int D>
struct FwdCfg {
    static constexpr int BM = 128;                 // rows per query tile (= TMEM lanes)
    static constexpr int TILES = 2;                // query tiles per work item
    static constexpr int BN = 128;                 // keys per K/V tile
    static constexpr int CHUNKS = D / 64;          // 64-element (128-byte) swizzle chunks per row
    static constexpr int Q_TILE_BYTES = BM * D * 2;
    static constexpr int TILE_BYTES = BN * D * 2;  // one K or V tile
    static constexpr int SLOTS = (D == 128) ? 4 : 10;
    static constexpr int STAGE_O_BYTES = 32 * 64 * 2;  // per softmax warp: 32 rows x 64 bf16
    static constexpr int NUM_THREADS = 384;
    static constexpr int NUM_PRODUCERS = 2;
    static constexpr int ITEM_RING = 4;  // work items handed from the fetching thread to the other roles
    // q_full, q_empty, slot_full, slot_empty, s_full, p_full, o_done, o_free, turn, drain, p_half,
    // item_full, item_empty, merge
    static constexpr int NUM_BARRIERS = 2 * 2 + 2 * (SLOTS + 1) + 7 * 2 + 2 * ITEM_RING + 1;
    // item readers: the second producer, the two MMA issuers and the eight softmax warps
    static constexpr int ITEM_READERS = 11;
    static constexpr int SMEM_BYTES = 1024 + TILES * Q_TILE_BYTES + SLOTS * TILE_BYTES + 8 * STAGE_O_BYTES +
                                      NUM_BARRIERS * 8 + 16 + ITEM_RING * 4;
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr float RESCALE_THRESHOLD = 8.0f;  // log2 units: P <= 2^8 between rescales
};

// The r-th item of this CTA in the static deal: rounds of gridDim.x items, dealt
// forwards in even rounds and backwards in odd ones. Past the last item of this
// CTA every later round is past the end too.
__device__ __forceinline__ int fwd_work_index(int r) {
    const int G = gridDim.x, c = blockIdx.x;
    return r * G + ((r & 1) ? (G - 1 - c) : c);
}

// One work item: a 256-row query block of one (batch, head), query tile t taking
// rows row0[t] .. row0[t] + 127 against key tiles 0 .. nk_t - 1. The items of a
// split launch (the SPLIT kernels, used for the last round of a non-causal
// problem) are 128-row halves of blocks: both query tiles take the same rows,
// tile 0 against key tiles [0, nk0) and tile 1 against [kb1, kb1 + nk1), and the
// two partial results are merged in the epilogue.
struct FwdItem {
    int qb, bh, b, h, hk;
    int nk0, nk1;  // key tiles of query tile 0 and 1 (nk1 - nk0 is 0 or 1)
    int row0[2];   // first query row of each tile
    int kb1;       // first key tile of tile 1 (0 unless split)
    bool split;
};

template <bool CAUSAL, bool SPLIT>
__device__ __forceinline__ FwdItem fwd_item(const FwdParams& p, int w) {
    FwdItem it;
    int half = 0;  // split items: which 128-row half of the block
    if (SPLIT) {
        half = w & 1;
        w = p.block0 + (w >> 1);
    }
    if (CAUSAL) {
        // heaviest blocks first: every (batch, head) at the last query block, then
        // at the one before, ...
        const int bh_count = p.B * p.Hq;
        it.bh = w % bh_count;
        it.qb = p.n_qblocks - 1 - w / bh_count;
    } else {
        // head by head: the query blocks of one head run in the same wave and
        // read its K/V tiles from L2
        it.bh = w / p.n_qblocks;
        it.qb = w % p.n_qblocks;
    }
    it.b = it.bh / p.Hq;
    it.h = it.bh % p.Hq;
    it.hk = it.h / (p.Hq / p.Hkv);
    const int n_kv = (p.N + 127) / 128;
    it.split = SPLIT;
    if (SPLIT) {
        it.nk0 = n_kv / 2;
        it.nk1 = n_kv - it.nk0;
        it.kb1 = it.nk0;
        it.row0[0] = it.row0[1] = it.qb * 256 + half * 128;
    } else {
        it.nk0 = CAUSAL ? min(2 * it.qb + 1, n_kv) : n_kv;
        it.nk1 = CAUSAL ? min(2 * it.qb + 2, n_kv) : n_kv;
        it.kb1 = 0;
        it.row0[0] = it.qb * 256;
        it.row0[1] = it.qb * 256 + 128;
    }
    return it;
}

// K/V loads of an item, in the order the producers issue them. A whole item
// streams K_0 V_0 K_1 V_1 ... for both tiles. A split item's loads each serve one
// tile, in the order its two MMA issuers consume them: K_0 of tile 0 and of tile
// 1, then per key step s the V_s and K_(s+1) of tile 0, then those of tile 1
// (leaving out what does not exist), so that a slot is never held up behind the
// other tile's later release.
__device__ __forceinline__ int fwd_item_loads(const FwdItem& it) { return 2 * (it.split ? it.nk0 + it.nk1 : it.nk1); }
// Load index (within the item) of K (v = false) or V (v = true) of query tile t's
// key step j. For a split item with h = nk0: V_t(s) = 2 + 4s + 2t and K_t(s+1)
// right after it while s + 1 < h; V_0(h-1), V_1(h-1) follow at 4h-2, 4h-1, then
// tile 1's extra step (nk1 = h + 1) has K_1(h) at 4h and V_1(h) at 4h+1.
__device__ __forceinline__ int fwd_load_index(const FwdItem& it, int t, int j, bool v) {
    if (!it.split) return 2 * j + (v ? 1 : 0);
    const int h = it.nk0;
    if (v) {
        if (j < h - 1) return 2 + 4 * j + 2 * t;
        return j == h - 1 ? 4 * h - 2 + t : 4 * h + 1;
    }
    if (j == 0) return t;
    if (j < h) return 3 + 4 * (j - 1) + 2 * t;
    return 4 * h;  // K_1(h)
}
// Load i of the item: whether it is a V tile, and its key tile.
__device__ __forceinline__ bool fwd_load_kind(const FwdItem& it, int i, int* key_tile) {
    if (!it.split) {
        *key_tile = i >> 1;
        return (i & 1) != 0;
    }
    const int h = it.nk0;
    int t, step;
    bool v;
    if (i < 2) {
        t = i; step = 0; v = false;
    } else if (i < 4 * h - 2) {
        const int s = (i - 2) >> 2, r = (i - 2) & 3;
        t = r >> 1; v = (r & 1) == 0; step = v ? s : s + 1;
    } else if (i < 4 * h) {
        t = i - (4 * h - 2); step = h - 1; v = true;
    } else {
        t = 1; step = h; v = i == 4 * h + 1;
    }
    *key_tile = step + (t ? it.kb1 : 0);
    return v;
}

// Max of 64 values with eight independent chains of 3-input max.
__device__ __forceinline__ float max64(const float (&v)[64]) {
    float m[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) m[k] = max3(v[k], v[8 + k], v[16 + k]);
#pragma unroll
    for (int k = 0; k < 8; ++k) m[k] = max3(m[k], v[24 + k], v[32 + k]);
#pragma unroll
    for (int k = 0; k < 8; ++k) m[k] = max3(m[k], v[40 + k], v[48 + k]);
#pragma unroll
    for (int k = 0; k < 8; ++k) m[k] = fmaxf(m[k], v[56 + k]);
    return max3(max3(m[0], m[1], m[2]), max3(m[3], m[4], m[5]), fmaxf(m[6], m[7]));
}

template <int D, bool CAUSAL, bool F32OUT, class E, bool SPLIT>
__global__ void __launch_bounds__(384, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                    const FwdParams p) {
    using C = FwdCfg<D>;
    constexpr int BM = C::BM, BN = C::BN;
    // split launches: both query tiles read Q buffer 0, and Q buffer 1 is a fifth
    // ring slot (a split item's K/V tiles each serve one tile: four loads a step)
    constexpr int SLOTS = C::SLOTS + (SPLIT ? 1 : 0);
    static_assert(C::Q_TILE_BYTES == C::TILE_BYTES, "the extra slot is a Q buffer");
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = smem;
    uint8_t* sKV = smem + C::TILES * C::Q_TILE_BYTES;
    uint8_t* sO = sKV + C::SLOTS * C::TILE_BYTES;  // [8 warps][32 rows][64 bf16] epilogue staging
    auto slot_ptr = [&](int slot) -> uint8_t* {
        return slot < C::SLOTS ? sKV + slot * C::TILE_BYTES : sQ + C::Q_TILE_BYTES;
    };
    uint64_t* bars = reinterpret_cast<uint64_t*>(sO + 8 * C::STAGE_O_BYTES);
    uint64_t* q_full = bars;                   // [2] Q tile t loaded
    uint64_t* q_empty = q_full + 2;            // [2] last S of Q tile t's buffer done
    uint64_t* slot_full = q_empty + 2;         // [SLOTS]
    uint64_t* slot_empty = slot_full + SLOTS;  // [SLOTS]
    uint64_t* s_full = slot_empty + SLOTS;     // [2] S_t ready
    uint64_t* p_full = s_full + 2;             // [2] P_t written (4 warp arrivals)
    uint64_t* o_done = p_full + 2;             // [2] a P V product complete
    uint64_t* o_free = o_done + 2;             // [2] epilogue has read O_t (4 warp arrivals)
    uint64_t* turn = o_free + 2;               // [2] softmax ping-pong (4 warp arrivals)
    uint64_t* drain = turn + 2;                // [2]
    uint64_t* p_half = drain + 2;              // [2] first half of P_t written (4 warp arrivals)
    uint64_t* item_full = p_half + 2;          // [ITEM_RING] work item r published
    uint64_t* item_empty = item_full + C::ITEM_RING;  // [ITEM_RING] read by every role (ITEM_READERS arrivals)
    uint64_t* merge_bar = item_empty + C::ITEM_RING;  // split item: tile 0's row max and sum published (4 warps)
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(merge_bar + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
    volatile int* item_ring = reinterpret_cast<volatile int*>(tmem_holder + 4);  // [ITEM_RING]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int t = 0; t < 2; ++t) {
            mbar_init(&q_full[t], C::CHUNKS);  // one expect_tx arrival per box
            mbar_init(&q_empty[t], 1);
            mbar_init(&s_full[t], 1);
            mbar_init(&p_full[t], 4);
            mbar_init(&o_done[t], 1);
            mbar_init(&o_free[t], 4);
            mbar_init(&turn[t], 4);
            mbar_init(&drain[t], 1);
            mbar_init(&p_half[t], 4);
        }
        for (int i = 0; i < SLOTS; ++i) {
            mbar_init(&slot_full[i], C::CHUNKS);
            mbar_init(&slot_empty[i], 2);  // released by both query tiles' MMAs
        }
        for (int i = 0; i < C::ITEM_RING; ++i) {
            mbar_init(&item_full[i], 1);
            mbar_init(&item_empty[i], C::ITEM_READERS);
        }
        if (SPLIT) mbar_init(merge_bar, 4);
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
    // The previous kernel's writes are visible after this wait. A split launch
    // that follows the launch of the same call's other blocks does not read
    // their outputs, and it is scheduled only once every block of that launch
    // has passed this wait (their trigger follows it), so its inputs are
    // complete: its blocks start on the SMs that launch's tail frees and wait
    // for it only before they exit, which keeps the stream's order of completion.
    const bool wait_at_end = SPLIT && p.chained;
    if (!wait_at_end) grid_dep_wait();

    // Work item r of this CTA: published by the first producer's thread (the
    // first item is the CTA's index, later ones come from the launch's counter,
    // taken while the previous item's last loads are issued so that the atomic's
    // latency hides behind them; p.n_items marks the end), read by every other
    // role in the same order. Returns the item, or -1 when a wait was abandoned.
    auto take_item = [&]() -> int {
        return static_cast<int>(gridDim.x + atomicAdd(&g_fwd_sched[p.sched_slot][0], 1u));
    };
    auto publish_item = [&](int r, int w) -> int {
        const int s = r % C::ITEM_RING;
        if (r >= C::ITEM_RING && !mbar_wait(&item_empty[s], ((r / C::ITEM_RING) - 1) & 1, abort_flag)) return -1;
        if (w > p.n_items) w = p.n_items;
        item_ring[s] = w;
        mbar_arrive(&item_full[s]);
        return w;
    };
    auto read_item = [&](int r) -> int {  // one thread: the second producer, an MMA issuer
        const int s = r % C::ITEM_RING;
        if (!mbar_wait(&item_full[s], (r / C::ITEM_RING) & 1, abort_flag)) return -1;
        const int w = item_ring[s];
        mbar_arrive(&item_empty[s]);
        return w;
    };
    auto read_item_warp = [&](int r) -> int {  // all 32 lanes of a softmax warp
        const int s = r % C::ITEM_RING;
        const bool ok_w = mbar_wait(&item_full[s], (r / C::ITEM_RING) & 1, abort_flag);
        const int w = item_ring[s];
        __syncwarp();
        if (lane == 0) mbar_arrive(&item_empty[s]);
        return __all_sync(0xffffffffu, ok_w) ? w : -1;
    };

    if (warp >= 10) {
        // ------------------------------------------------------ producers ---
        // Box c of Q tile t, and box c of K/V load g (K_j, V_j of an item are
        // loads base + 2j, base + 2j + 1), go to producer (index * CHUNKS + c) % 2;
        // each box arrives on its full barrier with its own byte count.
        if (lane == 0) {
            const int me = warp - 10;
            constexpr uint32_t BOX_BYTES = BN * 128;
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            bool ok = true;
            int g = 0, it = 0;
            int next_w = static_cast<int>(blockIdx.x);  // first producer: the item it publishes next
            for (int r = 0; ok; ++r, ++it) {
                const int w = CAUSAL ? fwd_work_index(r) : me == 0 ? publish_item(r, next_w) : read_item(r);
                if (w < 0) { ok = false; break; }
                if (w >= p.n_items) break;
                const FwdItem item = fwd_item<CAUSAL, SPLIT>(p, w);
                const int zq = item.b * p.Hq + item.h, zkv = item.b * p.Hkv + item.hk;
                // issue (this producer's boxes of) K/V load i of the item
                auto issue_kv = [&](int i) -> bool {
                    const int gi = g + i;
                    bool mine = false;
#pragma unroll
                    for (int c = 0; c < C::CHUNKS; ++c) mine |= ((gi * C::CHUNKS + c) % C::NUM_PRODUCERS) == me;
                    if (!mine) return true;
                    const int slot = gi % SLOTS, use = gi / SLOTS;
                    if (use > 0 && !mbar_wait_park(&slot_empty[slot], (use - 1) & 1, abort_flag)) return false;
                    int kt = i >> 1;
                    const CUtensorMap* tm = (i & 1) ? &tm_v : &tm_k;
                    if constexpr (SPLIT) tm = fwd_load_kind(item, i, &kt) ? &tm_v : &tm_k;
                    uint8_t* dst = slot_ptr(slot);
#pragma unroll
                    for (int c = 0; c < C::CHUNKS; ++c) {
                        if ((gi * C::CHUNKS + c) % C::NUM_PRODUCERS != me) continue;
                        mbar_arrive_expect_tx(&slot_full[slot], BOX_BYTES);
                        tma_load_3d(dst + c * BOX_BYTES, tm, &slot_full[slot], c * 64, kt * BN, zkv);
                    }
                    return true;
                };
                // issue (this producer's boxes of) Q tile t of the item
                auto issue_q = [&](int t) -> bool {
                    if (SPLIT && t == 1) return true;  // tile 1 reads Q buffer 0
                    bool any = false;
#pragma unroll
                    for (int c = 0; c < C::CHUNKS; ++c) any |= ((t * C::CHUNKS + c) % C::NUM_PRODUCERS) == me;
                    if (!any) return true;
                    if (it > 0 && !mbar_wait_park(&q_empty[t], (it - 1) & 1, abort_flag)) return false;
#pragma unroll
                    for (int c = 0; c < C::CHUNKS; ++c) {
                        if ((t * C::CHUNKS + c) % C::NUM_PRODUCERS != me) continue;
                        mbar_arrive_expect_tx(&q_full[t], BM * 128);
                        tma_load_3d(sQ + t * C::Q_TILE_BYTES + c * BM * 128, &tm_q, &q_full[t], c * 64,
                                    SPLIT ? item.row0[t] : item.qb * 2 * BM + t * BM, zq);
                    }
                    return true;
                };
                // Order: Q tile 0 (its buffer frees at tile 0's last S of the previous
                // item), K_0 and V_0 (slots the previous item's last tiles release),
                // then Q tile 1 (free after tile 1's last S, one key tile later in a
                // causal item), then the rest.
                // the first producer takes the next item two key tiles before this
                // item's last loads
                const int n_loads = SPLIT ? fwd_item_loads(item) : 2 * item.nk1;
                const int take_at = max(2, n_loads - 4);
                bool taken = false;
                ok = issue_q(0) && issue_kv(0) && issue_kv(1) && issue_q(1);
                for (int i = 2; ok && i < n_loads; ++i) {
                    if (!CAUSAL && me == 0 && i == take_at) {
                        next_w = take_item();
                        taken = true;
                    }
                    ok = issue_kv(i);
                }
                if (!CAUSAL && me == 0 && !taken) next_w = take_item();
                g += n_loads;
            }
            // Every load of this CTA is issued: the next kernel in the stream may be
            // scheduled (it waits for this grid's completion before reading memory).
            grid_dep_launch();
            // Let every copy in flight land before the CTA can exit.
            if (it > 0) {
                mbar_wait(&q_full[0], (it - 1) & 1, nullptr);
                if (!SPLIT) mbar_wait(&q_full[1], (it - 1) & 1, nullptr);
            }
            for (int i = max(0, g - SLOTS); i < g; ++i) mbar_wait(&slot_full[i % SLOTS], (i / SLOTS) & 1, nullptr);
        }
    } else if (warp >= 8) {
        // ---------------------------------------------------- MMA issuers ---
        const int t = warp - 8;
        if (lane == 0) {
            constexpr uint32_t idesc_qk = make_idesc(BM, BN, 0, 0, E::fmt);
            constexpr uint32_t idesc_pv = make_idesc(BM, D, 0, 1, E::fmt);
            const uint32_t s_tmem = tmem + t * 256, o_tmem = s_tmem + 128;
            const int tq = SPLIT ? 0 : t;  // the Q buffer this tile reads
            const uint32_t q_addr = smem_addr(sQ + tq * C::Q_TILE_BYTES), kv_addr = smem_addr(sKV);
            auto slot_addr = [&](int slot) -> uint32_t {
                return slot < C::SLOTS ? kv_addr + slot * C::TILE_BYTES : smem_addr(sQ + C::Q_TILE_BYTES);
            };
            bool ok = true;
            int g = 0;        // K/V load index of the item's K_0
            uint32_t np = 0;  // P_t handed over so far (p_full phases)
            for (int r = 0, it = 0; ok; ++r, ++it) {
                const int w = CAUSAL ? fwd_work_index(r) : read_item(r);
                if (w < 0) { ok = false; break; }
                if (w >= p.n_items) break;
                const FwdItem item = fwd_item<CAUSAL, SPLIT>(p, w);
                const int nk = t ? item.nk1 : item.nk0;
                // loads this tile alone uses: tile 1's extra key tile, and every load
                // of a split item; the other tile's release is given by hand
                auto single = [&](int jj) { return SPLIT || (t == 1 && jj >= item.nk0); };
                for (int j = 0; j <= nk; ++j) {
                    const int ik = SPLIT ? g + (j < nk ? fwd_load_index(item, t, j, false) : 0) : g + 2 * j;
                    const int iv = SPLIT ? g + (j > 0 ? fwd_load_index(item, t, j - 1, true) : 0) : g + 2 * j - 1;
                    if (j == 0) {
                        ok = mbar_wait(&q_full[tq], it & 1, abort_flag) &&
                             mbar_wait(&slot_full[ik % SLOTS], (ik / SLOTS) & 1, abort_flag);
                        if (!ok) break;
                        tc_fence_after();
                    } else {
                        // O_t += P_t(j-1) V_{j-1}. The loads (usually long done) are
                        // checked before P so only the wait for P is on the critical
                        // path; the first product of an item also needs the previous
                        // item's epilogue to have read O_t.
                        ok = mbar_wait(&slot_full[iv % SLOTS], (iv / SLOTS) & 1, abort_flag) &&
                             (j >= nk || mbar_wait(&slot_full[ik % SLOTS], (ik / SLOTS) & 1, abort_flag)) &&
                             (j > 1 || it == 0 || mbar_wait(&o_free[t], (it - 1) & 1, abort_flag)) &&
                             mbar_wait_spin(&p_half[t], np & 1, abort_flag);
                        if (!ok) break;
                        tc_fence_after();
                        const uint32_t v_addr = slot_addr(iv % SLOTS);
#pragma unroll
                        for (int kk = 0; kk < BN / 16; ++kk) {
                            if (kk == BN / 32) {
                                ok = mbar_wait_spin(&p_full[t], np & 1, abort_flag);
                                if (!ok) break;
                                tc_fence_after();
                            }
                            // V as the MN-major B operand: 16 keys = 2048 bytes per step;
                            // LBO = distance between the 64-column chunks of the tile.
                            const uint64_t bd = make_sdesc_sw128(v_addr + kk * 16 * 128, BN * 128, 1024);
                            mma_ts(o_tmem, s_tmem + kk * 8, bd, idesc_pv, (j > 1 || kk > 0) ? 1u : 0u);
                        }
                        if (!ok) break;
                        ++np;
                        if (j >= nk) {
                            tc_commit(&o_done[t]);
                            if (single(j - 1)) mbar_arrive(&slot_empty[iv % SLOTS]);
                            tc_commit(&slot_empty[iv % SLOTS]);
                            break;
                        }
                    }
                    // S_t(j) = Q_t K_j^T
                    const uint32_t k_addr = slot_addr(ik % SLOTS);
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t koff = (kk & 3) * 32;  // 16 elements = 32 bytes inside the swizzle row
                        const uint64_t ad = make_sdesc_sw128(q_addr + (kk >> 2) * (BM * 128) + koff, 16, 1024);
                        const uint64_t bd = make_sdesc_sw128(k_addr + (kk >> 2) * (BN * 128) + koff, 16, 1024);
                        mma_ss(s_tmem, ad, bd, idesc_qk, kk > 0 ? 1u : 0u);
                    }
                    tc_commit(&s_full[t]);
                    // P V(j-1) is signalled after S(j) so that the softmax hears of
                    // S first; each commit covers every earlier MMA of this thread.
                    if (j > 0) {
                        tc_commit(&o_done[t]);
                        if (single(j - 1)) mbar_arrive(&slot_empty[iv % SLOTS]);
                        tc_commit(&slot_empty[iv % SLOTS]);
                    }
                    if (single(j)) mbar_arrive(&slot_empty[ik % SLOTS]);
                    tc_commit(&slot_empty[ik % SLOTS]);
                    // Q_t's buffer is free once this S is done (split launches take one
                    // item per CTA: their Q buffer is never reloaded)
                    if (j == nk - 1 && !(SPLIT && t == 1)) tc_commit(&q_empty[t]);
                }
                g += SPLIT ? fwd_item_loads(item) : 2 * item.nk1;
            }
            // Every MMA must be complete before TMEM is released.
            tc_commit(&drain[t]);
            mbar_wait(&drain[t], 0, nullptr);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------- softmax ----
        const int t = warp >> 2;
        const int quad = warp & 3;  // TMEM lane quadrant this warp may access
        const int row = quad * 32 + lane;
        const uint32_t s_addr = tmem + t * 256 + (uint32_t(quad * 32) << 16);
        const uint32_t o_addr = s_addr + 128;
        const float c2 = p.scale_log2;
        bool ok = true;
        uint32_t ns = 0, nturn = 0, npv = 0, nmerge = 0;  // phases consumed so far, counted across items
        for (int r = 0; ok; ++r) {
            const int w = CAUSAL ? fwd_work_index(r) : read_item_warp(r);
            if (w < 0) { ok = false; break; }
            if (w >= p.n_items) break;
            const FwdItem item = fwd_item<CAUSAL, SPLIT>(p, w);
            const int nk = t ? item.nk1 : item.nk0;
            const int kb = (SPLIT && t) ? item.kb1 : 0;  // first key tile of this query tile
            const int grow = (SPLIT ? item.row0[t] : item.qb * 2 * BM + t * BM) + row;
            const int q128 = 2 * item.qb + t;  // index of this query tile in 128-row units (causal)
            float m_used = -INFINITY, l = 0.f;
            for (int j = 0; j < nk; ++j) {
                const bool w1 = mbar_wait(&s_full[t], ns & 1, abort_flag);
                if (!__all_sync(0xffffffffu, w1)) { ok = false; break; }
                ++ns;
                tc_fence_after();
                // valid key columns of this tile for this row: [0, lim)
                int lim = BN;
                if (CAUSAL && j == q128) lim = row + 1;
                if (!CAUSAL && (kb + j) * BN + BN > p.N) lim = p.N - (kb + j) * BN;
                // pass 1: row max
                float mx = -INFINITY;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    uint32_t r2[64];
                    tmem_ld64(s_addr + half * 64, r2);
                    if (__any_sync(0xffffffffu, half * 64 + 64 > lim)) {
#pragma unroll
                        for (int i = 0; i < 64; ++i)
                            if (half * 64 + i >= lim) r2[i] = 0xff800000u;  // -inf
                    }
                    mx = fmaxf(mx, max64(reinterpret_cast<const float(&)[64]>(r2)));
                }
                const float m_tile = mx * c2;
                const bool need = m_tile > m_used + C::RESCALE_THRESHOLD;
                float factor = 1.f;
                if (need) {
                    factor = ex2_approx(m_used - m_tile);
                    m_used = m_tile;
                }
                l *= factor;
                // S_t(j) completing implies O_t already holds every earlier P V
                // product, so O_t can be rescaled now, before P_t(j) is released.
                if (j > 0 && __any_sync(0xffffffffu, need)) {
#pragma unroll
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t r3[32];
                        tmem_ld32(o_addr + c * 32, r3);
#pragma unroll
                        for (int i = 0; i < 32; ++i) r3[i] = __float_as_uint(__uint_as_float(r3[i]) * factor);
                        tmem_st32(o_addr + c * 32, r3);
                    }
                }
                // The two softmax warpgroups take turns for the exp2 pass: tile 0 of
                // key tile j, then tile 1 of j, then tile 0 of j+1, ..., across items
                // too. Each then has the SFU to itself and the two tiles' MMAs
                // interleave with it; strict alternation also keeps every turn
                // barrier within one phase of its waiter. Tile 1's extra causal key
                // tile (the diagonal one of its rows) takes no turn: it overlaps
                // tile 0's first key tile of the next item.
                const bool my_turn_wait = (t == 0) ? (r > 0 || j > 0) : (j < item.nk0);
                if (my_turn_wait) {
                    const bool wt = mbar_wait(&turn[t], nturn & 1, abort_flag);
                    if (!__all_sync(0xffffffffu, wt)) { ok = false; break; }
                    ++nturn;
                }
                // pass 2: p = exp2(s * c2 - m), l += sum p, P (bf16) over the S columns.
                // Rows of a tile with no masked column (every warp of a non-diagonal,
                // non-tail tile) take a path with no per-element selects.
                const bool full = __all_sync(0xffffffffu, lim == BN);
                const float2 c2x2 = make_float2(c2, c2), negm2 = make_float2(-m_used, -m_used);
                float2 rsum[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) rsum[k] = make_float2(0.f, 0.f);
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    uint32_t r2[64];
                    tmem_ld64(s_addr + half * 64, r2);
                    if (!full) {
#pragma unroll
                        for (int i = 0; i < 64; ++i)
                            if (half * 64 + i >= lim) r2[i] = 0xff800000u;  // -inf: exp2 gives 0
                    }
                    uint32_t pk[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const float2 y = ffma2(make_float2(__uint_as_float(r2[2 * i]), __uint_as_float(r2[2 * i + 1])),
                                               c2x2, negm2);
                        const float2 pp = make_float2(ex2_approx(y.x), ex2_approx(y.y));
                        rsum[i & 3] = fadd2(rsum[i & 3], pp);
                        pk[i] = E::pack2(pp.x, pp.y);
                    }
                    tmem_st32(s_addr + half * 32, pk);
                    if (half == 0) {
                        // keys 0-63 of P_t are in TMEM: their P V steps may start
                        tmem_st_wait();
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&p_half[t]);
                    }
                }
                const float2 rs = fadd2(fadd2(rsum[0], rsum[1]), fadd2(rsum[2], rsum[3]));
                l += rs.x + rs.y;
                // pass the turn on: tile 0 always hands over to tile 1 of the same key
                // tile; tile 1 hands back after each key tile it shares with tile 0
                // (for key tile j + 1 of this item, or key tile 0 of the next item;
                // after the CTA's last item nobody waits for that turn)
                const bool hand_over = (t == 0) || (j < item.nk0);
                if (hand_over && lane == 0) mbar_arrive(&turn[1 - t]);
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();  // every lane's P stores precede the warp's one arrival
                if (lane == 0) mbar_arrive(&p_full[t]);
            }
            if (!ok) break;
            // Epilogue. PV(nk-2) is complete (S(nk-1) was seen; for nk = 1 the
            // previous item's epilogue waited for its last PV), so o_done is at
            // most one phase away and this parity wait is exact.
            npv += nk;
            const bool w2 = mbar_wait(&o_done[t], (npv - 1) & 1, abort_flag);
            if (!__all_sync(0xffffffffu, w2)) { ok = false; break; }
            tc_fence_after();
            // Split item: tile 0 hands this row's max and sum to tile 1 (through
            // its own staging buffer, whose last bulk store has read it) and leaves
            // its accumulator A_0 (the unnormalised sum of p v) in TMEM; tile 1
            // merges the two as the online softmax merges two blocks of keys,
            // O = (A_0 2^(m_0-M) + A_1 2^(m_1-M)) / (l_0 2^(m_0-M) + l_1 2^(m_1-M)) with
            // M = max(m_0, m_1), and frees A_0's columns once it has read them.
            float2* xch = reinterpret_cast<float2*>(sO + quad * C::STAGE_O_BYTES);
            if (SPLIT && t == 0) {
                if (lane == 0) bulk_wait_read_all();
                __syncwarp();
                xch[lane] = make_float2(m_used, l);
                __syncwarp();
                if (lane == 0) mbar_arrive(merge_bar);
                continue;
            }
            float m_fin = m_used, l_fin = l;
            if (SPLIT) {
                const bool wm = mbar_wait(merge_bar, nmerge & 1, abort_flag);
                ++nmerge;
                if (!__all_sync(0xffffffffu, wm)) { ok = false; break; }
                tc_fence_after();
                const float2 ml0 = xch[lane];
                m_fin = fmaxf(ml0.x, m_used);
                const float a0 = ex2_approx(ml0.x - m_fin), a1 = ex2_approx(m_used - m_fin);
                l_fin = ml0.y * a0 + l * a1;
                // A_1 <- A_1 2^(m_1-M) + A_0 2^(m_0-M), in TMEM; A_0 is then free
#pragma unroll 1
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t r3[32], r4[32];
                    tmem_ld32(o_addr + c * 32, r3);
                    tmem_ld32(o_addr - 256 + c * 32, r4);  // tile 0's O, same lanes
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        r3[i] = __float_as_uint(__uint_as_float(r3[i]) * a1 + __uint_as_float(r4[i]) * a0);
                    tmem_st32(o_addr + c * 32, r3);
                }
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&o_free[0]);
            }
            const float inv_l = 1.f / l_fin;
            uint8_t* stage = sO + warp * C::STAGE_O_BYTES;
            const int row0 = (SPLIT ? item.row0[t] : item.qb * 2 * BM + t * BM) + quad * 32;  // first row of this warp
            if constexpr (F32OUT) {
                // fp32 O, 32 columns (128 bytes of a row) at a time; chunk i of row
                // r sits at slot i ^ (r & 7) of the staging buffer
                float* of = static_cast<float*>(p.o);
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t r3[32];
                    tmem_ld32(o_addr + c * 32, r3);
                    if (c == D / 32 - 1) {
                        // O_t is in registers: the next item's first P V may overwrite it
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&o_free[t]);
                    }
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        *reinterpret_cast<float4*>(stage + lane * 128 + ((i ^ (lane & 7)) << 4)) =
                            make_float4(__uint_as_float(r3[4 * i + 0]) * inv_l, __uint_as_float(r3[4 * i + 1]) * inv_l,
                                        __uint_as_float(r3[4 * i + 2]) * inv_l, __uint_as_float(r3[4 * i + 3]) * inv_l);
                    __syncwarp();
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const int rr = 4 * k + (lane >> 3), chunk = lane & 7;
                        const float4 v4 = *reinterpret_cast<const float4*>(stage + rr * 128 + ((chunk ^ (rr & 7)) << 4));
                        if (row0 + rr < p.N)
                            *reinterpret_cast<float4*>(of + (static_cast<size_t>(item.bh) * p.N + row0 + rr) * D +
                                                       c * 32 + chunk * 4) = v4;
                    }
                    __syncwarp();
                }
            } else {
#pragma unroll
            for (int half = 0; half < D / 64; ++half) {
                // this lane's row, columns [64*half, 64*half + 64), read and rounded
                // before waiting for the staging buffer, so the TMEM loads overlap
                // the previous bulk store's read of it
                uint4 v4[8];
#pragma unroll
                for (int c2 = 0; c2 < 2; ++c2) {
                    const int c = half * 2 + c2;
                    uint32_t r3[32];
                    tmem_ld32(o_addr + c * 32, r3);
                    if (c == D / 32 - 1) {
                        // O_t is in registers: the next item's first P V may overwrite it
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&o_free[t]);
                    }
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        v4[c2 * 4 + i] = make_uint4(
                            E::pack2(__uint_as_float(r3[8 * i + 0]) * inv_l, __uint_as_float(r3[8 * i + 1]) * inv_l),
                            E::pack2(__uint_as_float(r3[8 * i + 2]) * inv_l, __uint_as_float(r3[8 * i + 3]) * inv_l),
                            E::pack2(__uint_as_float(r3[8 * i + 4]) * inv_l, __uint_as_float(r3[8 * i + 5]) * inv_l),
                            E::pack2(__uint_as_float(r3[8 * i + 6]) * inv_l, __uint_as_float(r3[8 * i + 7]) * inv_l));
                }
                // the staging buffer is free once the bulk store that read it last is done
                if (lane == 0) bulk_wait_read_all();
                __syncwarp();
                // 128 bytes as 8 chunks of 16; chunk i of row r sits at slot i ^ (r & 7),
                // the layout of a 128-byte-swizzled 32-row box of O
#pragma unroll
                for (int chunk = 0; chunk < 8; ++chunk)
                    *reinterpret_cast<uint4*>(stage + lane * 128 + ((chunk ^ (lane & 7)) << 4)) = v4[chunk];
                // one bulk tensor store of the warp's 32 rows x 64 columns (rows past N
                // are clipped by the tensor map); the warp goes on at once
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    tma_store_3d(&tm_o, stage, half * 64, row0, item.bh);
                    bulk_commit();
                }
            }
            }
            if (grow < p.N)
                p.lse[static_cast<size_t>(item.bh) * p.N + grow] = (m_fin + log2f(l_fin)) * 0.69314718055994530942f;
        }
        // the bulk stores read the staging buffers: complete before the CTA exits
        if (!F32OUT && lane == 0) bulk_wait_all();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 8) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
    if (wait_at_end) grid_dep_wait();
    // Every item this CTA took has been taken; the last CTA to get here resets the
    // launch's counter slot (no CTA of this launch reads it any more).
    if (!CAUSAL && threadIdx.x == 0) {
        unsigned int* ctr = g_fwd_sched[p.sched_slot];
        __threadfence();
        if (atomicAdd(&ctr[1], 1u) == gridDim.x - 1) {
            atomicExch(&ctr[0], 0u);
            atomicExch(&ctr[1], 0u);
        }
    }
}

}  // namespace eab
