// C ABI of the exact-attention library (declared in include/attn.h).
//
// Every call checks its arguments on the host before anything is enqueued,
// encodes the TMA tensor maps it needs (cuTensorMapEncodeTiled, fetched through
// the runtime's driver entry point so the library does not link libcuda), and
// launches on the caller's stream. The whole library is one translation unit so
// that the kernels share a single device-side status word.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <utility>
#include <cmath>
#include <cstdint>
#include <mutex>

#include "../../include/attn.h"
#include "attn_fwd_sm100.cuh"
#include "bwd_sm100.cuh"
#include "fp8_sm100.cuh"
#include "decode_sm100.cuh"
#include "merge_sm100.cuh"

namespace eab {
namespace {

// Launch with programmatic stream serialization: the kernel's blocks may be
// scheduled while the previous kernel in the stream is finishing (once all of
// its blocks have issued griddepcontrol.launch_dependents or exited); every
// kernel launched this way calls grid_dep_wait() before its first global
// memory access, so the order of the stream's memory effects is unchanged.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}


typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

// bf16 tensor viewed as [planes, rows, D] with a {64, box_rows, 1} box and
// 128-byte swizzle; rows past `rows` read as zero.
template <class E>
constexpr CUtensorMapDataType tma_type() {
    return E::fmt == ElemF16::fmt ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
}

template <class E>
bool make_map(CUtensorMap* map, const void* base, int D, int rows, int planes, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {cuuint64_t(D), cuuint64_t(rows), cuuint64_t(planes)};
    const cuuint64_t strides[2] = {cuuint64_t(D) * 2, cuuint64_t(D) * 2 * cuuint64_t(rows)};
    const cuuint32_t box[3] = {64, cuuint32_t(box_rows), 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(map, tma_type<E>(), 3, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// uint8 (E4M3 codes) tensor viewed as [planes, rows, inner] bytes with a
// {128, 128, 1} box and 128-byte swizzle; rows past `rows` read as zero.
bool make_map_u8(CUtensorMap* map, const void* base, int inner, int rows, int planes) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {cuuint64_t(inner), cuuint64_t(rows), cuuint64_t(planes)};
    const cuuint64_t strides[2] = {cuuint64_t(inner), cuuint64_t(inner) * cuuint64_t(rows)};
    const cuuint32_t box[3] = {128, 128, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool aligned16(const void* ptr) { return ptr != nullptr && (reinterpret_cast<uintptr_t>(ptr) & 15) == 0; }

bool scale_ok(float s) { return std::isfinite(s) && s > 0.f; }

constexpr float kLog2e = 1.4426950408889634f;

// The combine keeps one weight per split in dynamic shared memory; with its few
// static words it must stay under the 48 KiB a launch gets without opting in.
constexpr int kCombineMaxSplits = 12000;
// Longest sequence (N or L) a call accepts: counts rounded up to 256-row blocks
// or 128-key tiles (N + 255, L + S - 1, ...) then stay within int.
constexpr int kMaxSeq = 0x7fffffff - 255;

template <int D, bool CAUSAL, bool F32OUT, class E, bool SPLIT>
attn_status_t launch_fwd_kernel(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                                const CUtensorMap& to, const FwdParams& p, int grid, cudaStream_t stream) {
    using C = FwdCfg<D>;
    auto kern = attn_fwd_kernel<D, CAUSAL, F32OUT, E, SPLIT>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) != cudaSuccess)
        return ATTN_ERR_CUDA;
    if (launch_pdl(kern, dim3(grid), dim3(C::NUM_THREADS), C::SMEM_BYTES, stream, tq, tk, tv, to, p) != cudaSuccess)
        return ATTN_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

// Non-causal launches count their work items in a device counter slot; successive
// launches take successive slots (shared by every element type and output kind).
std::atomic<unsigned int> g_fwd_launch_seq{0};
int next_fwd_slot() { return static_cast<int>(g_fwd_launch_seq.fetch_add(1u) % kFwdSchedSlots); }

template <int D, bool CAUSAL, bool F32OUT, class E>
attn_status_t launch_fwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& to,
                         const FwdParams& p0, cudaStream_t stream) {
    // persistent grid: one CTA per SM, each walking its share of the work items
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1)
        return ATTN_ERR_CUDA;
    FwdParams p = p0;
    p.block0 = 0;
    p.chained = 0;
    if constexpr (!CAUSAL) {
        // Non-causal items all cost the same, so a last round of r <= SMs/2 query
        // blocks would leave most CTAs idle for a whole item. Those blocks go to a
        // second launch, right behind the first (programmatic dependent launch),
        // as two 128-row items each: both query tiles of a CTA on the same rows,
        // half of the key tiles each, merged at the end, so the last round takes
        // about half as long. Needs at least two key tiles.
        const int rem = p.n_items % sms;
        if ((p.N + 127) / 128 >= 2 && rem > 0 && 2 * rem <= sms) {
            const int n_full = p.n_items - rem;
            if (n_full > 0) {
                p.n_items = n_full;
                p.sched_slot = next_fwd_slot();
                const attn_status_t st = launch_fwd_kernel<D, CAUSAL, F32OUT, E, false>(tq, tk, tv, to, p, sms, stream);
                if (st != ATTN_OK) return st;
            }
            p.block0 = n_full;
            p.chained = n_full > 0 ? 1 : 0;
            p.n_items = 2 * rem;
            p.sched_slot = next_fwd_slot();
            return launch_fwd_kernel<D, CAUSAL, F32OUT, E, true>(tq, tk, tv, to, p, p.n_items, stream);
        }
        p.sched_slot = next_fwd_slot();
    }
    return launch_fwd_kernel<D, CAUSAL, F32OUT, E, false>(tq, tk, tv, to, p, p.n_items < sms ? p.n_items : sms,
                                                          stream);
}

template <int D, class E>
attn_status_t launch_decode(const CUtensorMap& tk, const CUtensorMap& tv, const DecodeParams& p, cudaStream_t stream) {
    using C = DecCfg<D>;
    auto kern = decode_splitkv_kernel<D, E>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) != cudaSuccess)
        return ATTN_ERR_CUDA;
    const dim3 grid(p.S, p.Hkv * p.groups, p.B);
    if (launch_pdl(kern, grid, dim3(C::NUM_THREADS), C::SMEM_BYTES, stream, tk, tv, p) != cudaSuccess)
        return ATTN_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

constexpr int kDecodeKeysSlots = 3;  // K/V ring of the keys-as-rows decode (3 slots: two blocks per SM)

template <int NQ, class E>
attn_status_t launch_decode_keys(const CUtensorMap& tk, const CUtensorMap& tv, const DecodeParams& p,
                                 cudaStream_t stream) {
    using C = DecTCfg<NQ, kDecodeKeysSlots>;
    auto kern = decode_splitkv_keys_kernel<NQ, kDecodeKeysSlots, E>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) != cudaSuccess)
        return ATTN_ERR_CUDA;
    const dim3 grid(p.S, p.Hkv, p.B);
    if (launch_pdl(kern, grid, dim3(C::NUM_THREADS), C::SMEM_BYTES, stream, tk, tv, p) != cudaSuccess)
        return ATTN_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

// One thread waits on an mbarrier that nothing completes, with a short limit.
__global__ void selftest_wait_kernel(uint64_t limit_ns) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
    mbar_wait(&bar, 0, &abort_flag, limit_ns);
}

template <bool F32OUT, class E>
attn_status_t fwd_impl(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                       int N, int d, int causal, float scale, attn_stream_t stream) {
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
        return ATTN_ERR_INVALID_ARG;
    if (B < 1 || Hq < 1 || Hkv < 1 || N < 1 || N > kMaxSeq || Hq % Hkv != 0 || (causal != 0 && causal != 1) ||
        !scale_ok(scale))
        return ATTN_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
    if (static_cast<long long>(B) * Hq > 65535LL * 1024) return ATTN_ERR_INVALID_ARG;
    CUtensorMap tq, tk, tv, to;
    if (!make_map<E>(&tq, q, d, N, B * Hq, 128) || !make_map<E>(&tk, k, d, N, B * Hkv, 128) ||
        !make_map<E>(&tv, v, d, N, B * Hkv, 128))
        return ATTN_ERR_CUDA;
    // O as 32-row boxes for the epilogue's bulk stores (16-bit outputs; the fp32
    // output is written by the threads and does not use it)
    if (F32OUT) to = tq;
    else if (!make_map<E>(&to, o, d, N, B * Hq, 32)) return ATTN_ERR_CUDA;
    FwdParams p;
    p.o = o;
    p.lse = lse;
    p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.N = N;
    p.n_qblocks = (N + 255) / 256;
    const long long items = static_cast<long long>(p.n_qblocks) * B * Hq;
    if (items > 0x7fffffffLL) return ATTN_ERR_INVALID_ARG;
    p.n_items = static_cast<int>(items);
    p.scale_log2 = scale * kLog2e;
    p.sched_slot = 0;  // taken by launch_fwd for non-causal launches
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (d == 128)
        return causal ? launch_fwd<128, true, F32OUT, E>(tq, tk, tv, to, p, st)
                      : launch_fwd<128, false, F32OUT, E>(tq, tk, tv, to, p, st);
    return causal ? launch_fwd<64, true, F32OUT, E>(tq, tk, tv, to, p, st)
                  : launch_fwd<64, false, F32OUT, E>(tq, tk, tv, to, p, st);
}

template <int D, bool CAUSAL, bool DKDV>
attn_status_t launch_bwd_tile(const CUtensorMap& fa, const CUtensorMap& fb, const CUtensorMap& sa,
                              const CUtensorMap& sb, const BwdParams& p, cudaStream_t stream) {
    using C = BwdCfg<D>;
    auto kern = bwd_tile_kernel<D, CAUSAL, DKDV>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) != cudaSuccess)
        return ATTN_ERR_CUDA;
    const dim3 grid(p.B * (DKDV ? p.Hkv : p.Hq), (p.N + C::BT - 1) / C::BT);
    if (launch_pdl(kern, grid, dim3(C::NUM_THREADS), C::SMEM_BYTES, stream, fa, fb, sa, sb, p) != cudaSuccess)
        return ATTN_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

template <int D, bool CAUSAL>
attn_status_t launch_bwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                         const CUtensorMap& tdo, const BwdParams& p, cudaStream_t stream) {
    const long long rows = static_cast<long long>(p.B) * p.Hq * p.N;
    constexpr long long kRowsPerBlock = 256 / (D / 8);
    launch_pdl(bwd_delta_kernel<D>, dim3(static_cast<unsigned>((rows + kRowsPerBlock - 1) / kRowsPerBlock)), dim3(256),
               0, stream, p, rows);
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
    attn_status_t st = launch_bwd_tile<D, CAUSAL, true>(tk, tv, tq, tdo, p, stream);
    if (st != ATTN_OK) return st;
    return launch_bwd_tile<D, CAUSAL, false>(tq, tdo, tk, tv, p, stream);
}

template <class E>
attn_status_t decode_impl(const void* q, const void* k, const void* v, float* o_part, float* lse_part,
                                  int B, int Hq, int Hkv, int L, int d, int num_splits, float scale,
                                  attn_stream_t stream) {
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o_part) || !aligned16(lse_part))
        return ATTN_ERR_INVALID_ARG;
    if (B < 1 || Hq < 1 || Hkv < 1 || L < 1 || L > kMaxSeq || Hq % Hkv != 0 || num_splits < 1 ||
        num_splits > L || !scale_ok(scale))
        return ATTN_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
    if (B > 65535 || num_splits > 0x7fffffff / 2) return ATTN_ERR_INVALID_ARG;
    const int per = (L + num_splits - 1) / num_splits;
    const int chunk = (per + 127) / 128 * 128;  // whole 128-key tiles
    CUtensorMap tk, tv;
    if (!make_map<E>(&tk, k, d, L, B * Hkv, 128) || !make_map<E>(&tv, v, d, L, B * Hkv, 128)) return ATTN_ERR_CUDA;
    DecodeParams p;
    p.q = q;
    p.o_part = o_part;
    p.lse_part = lse_part;
    p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.L = L; p.S = num_splits; p.chunk = chunk;
    p.G = Hq / Hkv;
    p.groups = (p.G + 127) / 128;  // query heads of a KV head, 128 rows per block
    if (static_cast<long long>(Hkv) * p.groups > 65535) return ATTN_ERR_INVALID_ARG;
    p.scale_log2 = scale * kLog2e;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    // small groups at d = 128: keys as the tile rows (a few query heads cannot
    // fill 128 rows); other shapes: the query heads as the tile rows
    if (d == 128 && p.G <= 16) return launch_decode_keys<16, E>(tk, tv, p, st);
    if (d == 128 && p.G <= 32) return launch_decode_keys<32, E>(tk, tv, p, st);
    return d == 128 ? launch_decode<128, E>(tk, tv, p, st) : launch_decode<64, E>(tk, tv, p, st);
}

template <class E>
attn_status_t combine_impl(const float* o_part, const float* lse_part, void* o, float* lse, int B, int Hq,
                           int num_splits, int d, attn_stream_t stream) {
    if (!aligned16(o_part) || !aligned16(lse_part) || !aligned16(o) || !aligned16(lse)) return ATTN_ERR_INVALID_ARG;
    if (B < 1 || Hq < 1 || num_splits < 1) return ATTN_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
    const long long blocks = static_cast<long long>(B) * Hq;
    const size_t smem = static_cast<size_t>(num_splits) * sizeof(float);
    if (blocks > 0x7fffffffLL || num_splits > kCombineMaxSplits) return ATTN_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    auto* ob = static_cast<typename E::T*>(o);
    if (d == 128)
        launch_pdl(combine_kernel<128, E>, dim3(static_cast<unsigned>(blocks)), dim3(128), smem, st, o_part, lse_part,
                   ob, lse, num_splits);
    else
        launch_pdl(combine_kernel<64, E>, dim3(static_cast<unsigned>(blocks)), dim3(64), smem, st, o_part, lse_part,
                   ob, lse, num_splits);
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // namespace
}  // namespace eab

using namespace eab;

extern "C" {

const char* attn_status_string(attn_status_t s) {
    switch (s) {
        case ATTN_OK: return "ATTN_OK";
        case ATTN_ERR_INVALID_ARG: return "ATTN_ERR_INVALID_ARG";
        case ATTN_ERR_UNSUPPORTED: return "ATTN_ERR_UNSUPPORTED";
        case ATTN_ERR_CUDA: return "ATTN_ERR_CUDA";
        case ATTN_ERR_TIMEOUT: return "ATTN_ERR_TIMEOUT";
    }
    return "ATTN_ERR_UNKNOWN";
}

attn_status_t attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                       int N, int d, int causal, float scale, attn_stream_t stream) {
    return fwd_impl<false, ElemBf16>(q, k, v, o, lse, B, Hq, Hkv, N, d, causal, scale, stream);
}

attn_status_t attn_fwd_f32(const void* q, const void* k, const void* v, float* o, float* lse, int B, int Hq,
                           int Hkv, int N, int d, int causal, float scale, attn_stream_t stream) {
    return fwd_impl<true, ElemBf16>(q, k, v, o, lse, B, Hq, Hkv, N, d, causal, scale, stream);
}

attn_status_t attn_fwd_f16(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                           int N, int d, int causal, float scale, attn_stream_t stream) {
    return fwd_impl<false, ElemF16>(q, k, v, o, lse, B, Hq, Hkv, N, d, causal, scale, stream);
}

attn_status_t attn_decode_splitkv(const void* q, const void* k, const void* v, float* o_part, float* lse_part,
                                  int B, int Hq, int Hkv, int L, int d, int num_splits, float scale,
                                  attn_stream_t stream) {
    return decode_impl<ElemBf16>(q, k, v, o_part, lse_part, B, Hq, Hkv, L, d, num_splits, scale, stream);
}

attn_status_t attn_decode_splitkv_f16(const void* q, const void* k, const void* v, float* o_part, float* lse_part,
                                      int B, int Hq, int Hkv, int L, int d, int num_splits, float scale,
                                      attn_stream_t stream) {
    return decode_impl<ElemF16>(q, k, v, o_part, lse_part, B, Hq, Hkv, L, d, num_splits, scale, stream);
}

attn_status_t attn_combine(const float* o_part, const float* lse_part, void* o, float* lse, int B, int Hq,
                           int num_splits, int d, attn_stream_t stream) {
    return combine_impl<ElemBf16>(o_part, lse_part, o, lse, B, Hq, num_splits, d, stream);
}

attn_status_t attn_combine_f16(const float* o_part, const float* lse_part, void* o, float* lse, int B, int Hq,
                               int num_splits, int d, attn_stream_t stream) {
    return combine_impl<ElemF16>(o_part, lse_part, o, lse, B, Hq, num_splits, d, stream);
}

attn_status_t attn_merge(float* o_acc, float* lse_acc, const float* o_blk, const float* lse_blk, void* out,
                         long long rows, int d, int init, attn_stream_t stream) {
    if (!aligned16(o_acc) || !aligned16(lse_acc) || !aligned16(o_blk) || !aligned16(lse_blk)) return ATTN_ERR_INVALID_ARG;
    if (out != nullptr && !aligned16(out)) return ATTN_ERR_INVALID_ARG;
    if (rows < 1) return ATTN_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
    const long long blocks = (rows + 7) / 8;  // one warp per row, 8 rows per block
    if (blocks > 0x7fffffffLL) return ATTN_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    auto* outb = static_cast<__nv_bfloat16*>(out);
    if (d == 128)
        launch_pdl(merge_kernel<128>, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, st, o_acc, lse_acc, o_blk,
                   lse_blk, outb, rows, init);
    else
        launch_pdl(merge_kernel<64>, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, st, o_acc, lse_acc, o_blk,
                   lse_blk, outb, rows, init);
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

attn_status_t attn_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
                       const void* dout, float* delta, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int N,
                       int d, int causal, float scale, attn_stream_t stream) {
    const void* ptrs[] = {q, k, v, o, lse, dout, delta, dq, dk, dv};
    for (const void* ptr : ptrs)
        if (!aligned16(ptr)) return ATTN_ERR_INVALID_ARG;
    if (B < 1 || Hq < 1 || Hkv < 1 || N < 1 || N > kMaxSeq || Hq % Hkv != 0 || (causal != 0 && causal != 1) ||
        !scale_ok(scale))
        return ATTN_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
    // the tile kernels' grid is (planes, 128-row tiles): both within 65535
    if (static_cast<long long>(B) * Hq > 65535LL || (N + 127) / 128 > 65535) return ATTN_ERR_INVALID_ARG;
    if ((static_cast<long long>(B) * Hq * N + 7) / 8 > 0x7fffffffLL) return ATTN_ERR_INVALID_ARG;
    CUtensorMap tq, tk, tv, tdo;
    if (!make_map<ElemBf16>(&tq, q, d, N, B * Hq, 128) || !make_map<ElemBf16>(&tk, k, d, N, B * Hkv, 128) ||
        !make_map<ElemBf16>(&tv, v, d, N, B * Hkv, 128) || !make_map<ElemBf16>(&tdo, dout, d, N, B * Hq, 128))
        return ATTN_ERR_CUDA;
    BwdParams p;
    p.o = static_cast<const __nv_bfloat16*>(o);
    p.dout = static_cast<const __nv_bfloat16*>(dout);
    p.lse = lse;
    p.delta = delta;
    p.dq = static_cast<__nv_bfloat16*>(dq);
    p.dk = static_cast<__nv_bfloat16*>(dk);
    p.dv = static_cast<__nv_bfloat16*>(dv);
    p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.N = N;
    p.scale = scale;
    p.scale_log2 = scale * kLog2e;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (d == 128) return causal ? launch_bwd<128, true>(tq, tk, tv, tdo, p, st) : launch_bwd<128, false>(tq, tk, tv, tdo, p, st);
    return causal ? launch_bwd<64, true>(tq, tk, tv, tdo, p, st) : launch_bwd<64, false>(tq, tk, tv, tdo, p, st);
}

attn_status_t attn_quant_fp8(const void* x, void* codes, float* scales, int planes, int N, int d, int per_plane,
                             int transpose, attn_stream_t stream) {
    if (!aligned16(x) || !aligned16(codes) || !aligned16(scales)) return ATTN_ERR_INVALID_ARG;
    if (planes < 1 || N < 1 || N > kMaxSeq || (per_plane != 0 && per_plane != 1) ||
        (transpose != 0 && transpose != 1))
        return ATTN_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
    const int nblk = (N + 127) / 128;
    if (planes > 65535) return ATTN_ERR_INVALID_ARG;
    QuantParams p{};
    p.x = static_cast<const __nv_bfloat16*>(x);
    p.codes = static_cast<uint8_t*>(codes);
    p.scales = scales;
    p.planes = planes; p.N = N; p.nblk = nblk; p.Np = nblk * 128; p.per_plane = per_plane;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const dim3 grid(nblk, planes);
    if (!per_plane && !transpose) {
        // per-block scales, row-major codes: one pass over x
        if (d == 128) launch_pdl(fp8_quant_rows_kernel<128, false>, grid, dim3(kQuantRowsThreads), 0, st, p);
        else launch_pdl(fp8_quant_rows_kernel<64, false>, grid, dim3(kQuantRowsThreads), 0, st, p);
        return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
    }
    if (d == 128) {
        launch_pdl(fp8_amax_kernel<128>, grid, dim3(256), 0, st, p);
        if (transpose) launch_pdl(fp8_quant_kernel<128, true>, grid, dim3(256), 0, st, p);
        else launch_pdl(fp8_quant_kernel<128, false>, grid, dim3(256), 0, st, p);
    } else {
        launch_pdl(fp8_amax_kernel<64>, grid, dim3(256), 0, st, p);
        if (transpose) launch_pdl(fp8_quant_kernel<64, true>, grid, dim3(256), 0, st, p);
        else launch_pdl(fp8_quant_kernel<64, false>, grid, dim3(256), 0, st, p);
    }
    launch_pdl(fp8_scales_kernel, dim3((planes + 255) / 256), dim3(256), 0, st, p);
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

attn_status_t attn_quant_fp8_rotate(const void* x, const float* signs, void* codes, float* scales, int planes, int N,
                                    int d, attn_stream_t stream) {
    if (!aligned16(x) || !aligned16(signs) || !aligned16(codes) || !aligned16(scales)) return ATTN_ERR_INVALID_ARG;
    if (planes < 1 || N < 1 || N > kMaxSeq || planes > 65535) return ATTN_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
    const int nblk = (N + 127) / 128;
    QuantParams p{};
    p.x = static_cast<const __nv_bfloat16*>(x);
    p.codes = static_cast<uint8_t*>(codes);
    p.scales = scales;
    p.planes = planes; p.N = N; p.nblk = nblk; p.Np = nblk * 128; p.per_plane = 0;
    p.signs = signs;
    p.rot_scale = static_cast<float>(1.0 / std::sqrt(static_cast<double>(d)));
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const dim3 grid(nblk, planes);
    if (d == 128) launch_pdl(fp8_quant_rows_kernel<128, true>, grid, dim3(kQuantRowsThreads), 0, st, p);
    else launch_pdl(fp8_quant_rows_kernel<64, true>, grid, dim3(kQuantRowsThreads), 0, st, p);
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

attn_status_t attn_fwd_fp8(const void* q8, const void* k8, const void* vt8, const float* sq, const float* sk,
                           const float* sv, void* o, float* lse, int B, int Hq, int Hkv, int N, int d, int causal,
                           float scale, attn_stream_t stream) {
    const void* ptrs[] = {q8, k8, vt8, sq, sk, sv, o, lse};
    for (const void* ptr : ptrs)
        if (!aligned16(ptr)) return ATTN_ERR_INVALID_ARG;
    if (B < 1 || Hq < 1 || Hkv < 1 || N < 1 || N > kMaxSeq || Hq % Hkv != 0 || (causal != 0 && causal != 1) ||
        !scale_ok(scale))
        return ATTN_ERR_INVALID_ARG;
    if (d != 128) return ATTN_ERR_UNSUPPORTED;
    if (static_cast<long long>(B) * Hq > 65535LL) return ATTN_ERR_INVALID_ARG;
    const int nblk = (N + 127) / 128;
    CUtensorMap tq, tk, tv;
    if (!make_map_u8(&tq, q8, 128, N, B * Hq) || !make_map_u8(&tk, k8, 128, N, B * Hkv) ||
        !make_map_u8(&tv, vt8, nblk * 128, 128, B * Hkv))
        return ATTN_ERR_CUDA;
    Fp8Params p;
    p.sq = sq; p.sk = sk; p.sv = sv;
    p.o = static_cast<__nv_bfloat16*>(o);
    p.lse = lse;
    p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.N = N; p.nblk = nblk;
    p.scale_log2 = scale * kLog2e;
    p.n_qblocks = (N + 255) / 256;
    const long long items = static_cast<long long>(p.n_qblocks) * B * Hq;
    if (items > (1LL << 30)) return ATTN_ERR_INVALID_ARG;
    p.n_items = static_cast<int>(items);
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1)
        return ATTN_ERR_CUDA;
    // without the causal mask a grid of up to twice the items lets the kernel
    // deal 128-row halves to otherwise idle SMs
    const int want = (!causal && 2 * p.n_items <= sms) ? 2 * p.n_items : p.n_items;
    const int grid = want < sms ? want : sms;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    auto kern = causal ? attn_fwd_fp8_kernel<true> : attn_fwd_fp8_kernel<false>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Fp8Cfg::SMEM_BYTES) != cudaSuccess)
        return ATTN_ERR_CUDA;
    if (launch_pdl(kern, dim3(grid), dim3(Fp8Cfg::NUM_THREADS), Fp8Cfg::SMEM_BYTES, st, tq, tk, tv, p) != cudaSuccess)
        return ATTN_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

int attn_decode_default_splits(int B, int Hq, int Hkv, int L) {
    if (B < 1 || Hq < 1 || Hkv < 1 || L < 1 || L > kMaxSeq || Hq % Hkv != 0) return 0;
    // Decode blocks (one per SM, 148 on B200; two per SM for the keys-as-rows
    // kernel with a 3-slot ring) each stream their split at about their share of
    // HBM bandwidth after a fixed start-up worth ~260 keys. Pick the split count
    // that maximises (busy fraction of the block waves) x (streaming fraction
    // chunk / (chunk + 260)); splits are whole 128-key tiles.
    const int G = Hq / Hkv;
    const int kSMs = 148 * (G <= 32 ? DecTCfg<16, kDecodeKeysSlots>::BLOCKS_PER_SM : 1);
    constexpr int kStage = 128;
    constexpr double kStartupKeys = 260.0;
    const long long units = static_cast<long long>(B) * Hkv * ((G + 127) / 128);
    const int max_s = static_cast<int>(std::min<long long>((L + kStage - 1) / kStage, 4096));
    int best_s = 1;
    double best = -1.0;
    for (int S = 1; S <= max_s; ++S) {
        const long long per = (L + S - 1) / S;
        const long long chunk = (per + kStage - 1) / kStage * kStage;
        const long long nonempty = (L + chunk - 1) / chunk;
        const long long waves = (units * S + kSMs - 1) / kSMs;
        const double busy = static_cast<double>(units * nonempty) / static_cast<double>(kSMs * waves);
        const double score = busy * (chunk / (chunk + kStartupKeys));
        if (score > best + 1e-9) {
            best = score;
            best_s = S;
        }
    }
    return best_s;
}

attn_status_t attn_device_status(attn_stream_t stream) {
    if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return ATTN_ERR_CUDA;
    int value = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&value, g_attn_status, sizeof(int)) != cudaSuccess) return ATTN_ERR_CUDA;
    if (value != 0 && cudaMemcpyToSymbol(g_attn_status, &zero, sizeof(int)) != cudaSuccess) return ATTN_ERR_CUDA;
    return value == 0 ? ATTN_OK : static_cast<attn_status_t>(value);
}

attn_status_t attn_selftest_bounded_wait(int limit_us, attn_stream_t stream) {
    if (limit_us < 1 || limit_us > 1000000) return ATTN_ERR_INVALID_ARG;
    selftest_wait_kernel<<<1, 1, 0, reinterpret_cast<cudaStream_t>(stream)>>>(uint64_t(limit_us) * 1000ull);
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Decode without any device allocation by the caller or the library.
//
// Some callers cannot hand this library a scratch buffer for the split
// partials: code that runs where the device memory is already fully owned by
// another allocator (a serving engine's pre-reserved pool, a host application
// that forbids allocations from plug-ins), or latency-critical loops where a
// cudaMalloc and the device synchronisation it can imply are not acceptable.
// For them, attn_decode_noalloc keeps the partials in one fixed array compiled
// into the library: a file-scope __device__ array that every GPU which loads the
// library holds until the process exits.
namespace eab {
namespace {

constexpr size_t kNoAllocScratchFloats = size_t(1) << 20;  // 4 MiB per device
static __device__ __align__(256) float g_decode_scratch[kNoAllocScratchFloats];

// Host code only holds a stand-in for the array's name; the device address is
// looked up once per device (with that device current) and cached.
constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

attn_status_t scratch_for_current_device(float** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ATTN_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (g_scratch_ptr[dev] == nullptr) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_decode_scratch) != cudaSuccess || ptr == nullptr) return ATTN_ERR_CUDA;
        g_scratch_ptr[dev] = ptr;
    }
    *out = static_cast<float*>(g_scratch_ptr[dev]);
    return ATTN_OK;
}

}  // namespace
}  // namespace eab

extern "C" attn_status_t attn_decode_noalloc(const void* q, const void* k, const void* v, void* o, float* lse,
                                             int B, int Hq, int Hkv, int L, int d, int num_splits, float scale,
                                             attn_stream_t stream) {
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
        return ATTN_ERR_INVALID_ARG;
    if (B < 1 || Hq < 1 || Hkv < 1 || L < 1 || L > kMaxSeq || num_splits < 1 || num_splits > L)
        return ATTN_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
    // every limit of the two launches is checked here, so that nothing is
    // enqueued unless both can run
    if (num_splits > kCombineMaxSplits || Hq % Hkv != 0 || !scale_ok(scale) || B > 65535 ||
        static_cast<long long>(Hkv) * ((Hq / Hkv + 127) / 128) > 65535)
        return ATTN_ERR_INVALID_ARG;
    // partials: o_part [B,Hq,S,d] then lse_part [B,Hq,S], all fp32
    const unsigned long long units = static_cast<unsigned long long>(B) * Hq * num_splits;
    if (units * (static_cast<unsigned long long>(d) + 1) > kNoAllocScratchFloats) return ATTN_ERR_INVALID_ARG;
    float* scratch = nullptr;
    if (attn_status_t st = scratch_for_current_device(&scratch); st != ATTN_OK) return st;
    float* o_part = scratch;
    float* lse_part = scratch + units * d;  // d*4 bytes per unit keeps this 16-byte aligned
    if (attn_status_t st = attn_decode_splitkv(q, k, v, o_part, lse_part, B, Hq, Hkv, L, d, num_splits, scale,
                                               stream);
        st != ATTN_OK)
        return st;
    return attn_combine(o_part, lse_part, o, lse, B, Hq, num_splits, d, stream);
}
