// Ring attention (context parallelism): folding the attention of one key/value
// block into a running result.
//
// FlashAttention-3 page: attention over a key range that has been split into
// parts is the log-sum-exp weighted merge of the parts (its split-K combine,
// and the RingAttention derivation it refers to, where the key/value shards of
// a long sequence travel around a ring of devices). With
// M = max(lse_acc, lse_blk), wa = exp(lse_acc - M), wb = exp(lse_blk - M):
//   o_acc <- (wa * o_acc + wb * o_blk) / (wa + wb),   lse_acc <- M + ln(wa + wb).
//
// The block's O arrives in fp32 (attn_fwd_f32), so it is rounded to bf16 only
// once, by the last merge. The merge reads and writes every element once, so it
// is bound by HBM bandwidth: one warp per row, each lane owns D/32 consecutive
// columns (16-byte fp32 vectors at D = 128), 8 rows per 256-thread block.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

namespace eab {

template <int D>
__global__ void __launch_bounds__(256)
    merge_kernel(float* __restrict__ o_acc, float* __restrict__ lse_acc, const float* __restrict__ o_blk,
                 const float* __restrict__ lse_blk, __nv_bfloat16* __restrict__ out, long long rows, int init) {
    grid_dep_wait();  // the previous kernel's writes are visible from here on
    grid_dep_launch();
    constexpr int CPL = D / 32;  // columns per lane
    const long long row = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
    if (row >= rows) return;
    const int lane = threadIdx.x & 31;
    const size_t base = static_cast<size_t>(row) * D + lane * CPL;

    float b[CPL];
    if constexpr (CPL == 4) {
        const float4 u = *reinterpret_cast<const float4*>(o_blk + base);
        b[0] = u.x; b[1] = u.y; b[2] = u.z; b[3] = u.w;
    } else {
        const float2 u = *reinterpret_cast<const float2*>(o_blk + base);
        b[0] = u.x; b[1] = u.y;
    }
    const float lb = lse_blk[row];

    float a[CPL];
    float la;
    if (init) {
#pragma unroll
        for (int i = 0; i < CPL; ++i) a[i] = b[i];
        la = lb;
    } else {
        if constexpr (CPL == 4) {
            const float4 v = *reinterpret_cast<const float4*>(o_acc + base);
            a[0] = v.x; a[1] = v.y; a[2] = v.z; a[3] = v.w;
        } else {
            const float2 v = *reinterpret_cast<const float2*>(o_acc + base);
            a[0] = v.x; a[1] = v.y;
        }
        la = lse_acc[row];
        const float M = fmaxf(la, lb);
        if (M != -INFINITY) {  // both sides empty: the row stays (o_acc, -inf)
            const float wa = (la == -INFINITY) ? 0.f : expf(la - M);
            const float wb = (lb == -INFINITY) ? 0.f : expf(lb - M);
            const float inv = 1.f / (wa + wb);
#pragma unroll
            for (int i = 0; i < CPL; ++i) a[i] = (wa * a[i] + wb * b[i]) * inv;
            la = M + logf(wa + wb);
        }
    }

    if (out != nullptr) {
        if constexpr (CPL == 4) {
            const __nv_bfloat162 p0 = __floats2bfloat162_rn(a[0], a[1]), p1 = __floats2bfloat162_rn(a[2], a[3]);
            *reinterpret_cast<uint2*>(out + base) =
                make_uint2(*reinterpret_cast<const uint32_t*>(&p0), *reinterpret_cast<const uint32_t*>(&p1));
        } else {
            const __nv_bfloat162 p0 = __floats2bfloat162_rn(a[0], a[1]);
            *reinterpret_cast<__nv_bfloat162*>(out + base) = p0;
        }
    } else {
        if constexpr (CPL == 4)
            *reinterpret_cast<float4*>(o_acc + base) = make_float4(a[0], a[1], a[2], a[3]);
        else
            *reinterpret_cast<float2*>(o_acc + base) = make_float2(a[0], a[1]);
    }
    if (lane == 0) lse_acc[row] = la;
}

}  // namespace eab
