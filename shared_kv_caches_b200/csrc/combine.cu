// Combine pass of split-KV decoding: merge the per-part results of each
// (sequence, head[, branch]) by their log-sum-exp, sum the MLRA branches and
// cast to the output type.
//
// For parts p with normalised output o_p and lse_p, the whole context has
// lse = ln sum_p exp(lse_p) and o = sum_p exp(lse_p - lse) o_p.  The MLRA page
// (aitntnews.com newId=23265, "moving the sum outside") sums the branch
// outputs after attention: out[b,h] = sum_r o[b,h,r].  GLA group heads need no
// placement here: the decode kernels already write partial rows by global
// head index.
#include <math.h>

#include "kvattn_internal.cuh"

namespace kvattn {

namespace {

constexpr int kThreads = 128;
constexpr int kMaxV4 = kThreads;           // float4 columns a block can own

// Row groups per block.  With many (branch, part) rows (a long single
// sequence split over the whole GPU) 16 groups share them and a block owns 32
// value columns; otherwise a block owns the whole value row (up to 512
// columns) and the groups split what is left of the 128 threads.
__host__ __device__ inline int combine_groups(int rows, int dv)
{
    if (rows >= 64)
        return 16;
    const int v4 = dv / 4;
    return v4 >= kThreads ? 1 : kThreads / v4;
}

// One block per (head, sequence, chunk of value columns).  The pass is bound
// by memory latency, so every load that does not depend on another goes out
// first: each thread issues up to PRE of its partial rows (G groups of
// 128/G threads split the (branch, part) rows, a thread owning four value
// columns) while the block copies all the parts' lse values to shared memory
// in one pass; then one warp per branch turns them into merge weights, the
// threads finish their rows, and the groups meet in shared memory.
template <int PRE>
__global__ void __launch_bounds__(kThreads) combine_kernel(const CombineArgs a)
{
    extern __shared__ float w_s[];     // [R][S] lse, then merge weights
    __shared__ float4 acc_s[kMaxV4];
    const int h = blockIdx.x, b = blockIdx.y;
    const int R = a.mlra ? a.NU : 1;
    const int S = a.num_splits;
    const int rows = R * S;
    const int kGroups = combine_groups(rows, a.Dv);
    const int kV4 = kThreads / kGroups;
    const int c0 = blockIdx.z * 4 * kV4;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = tid / kV4, q4 = tid % kV4;
    pdl_wait_primary();        // the decode pass has finished and its parts are visible
    const int col = c0 + 4 * q4;
    const bool on = col < a.Dv;

    auto row_ptr = [&](int k) {
        const int r = k / S, s = k % S;
        const int hu = a.mlra ? h * R + r : h;
        return reinterpret_cast<const float4 *>(a.po + (((size_t)b * S + s) * a.HU + hu) * a.Dv + col);
    };
    float4 v[PRE];
#pragma unroll
    for (int u = 0; u < PRE; ++u) {
        const int k = g + u * kGroups;
        v[u] = (on && k < rows) ? __ldcs(row_ptr(k)) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    for (int k = tid; k < rows; k += kThreads) {
        const int r = k / S, s = k % S;
        const int hu = a.mlra ? h * R + r : h;
        w_s[k] = a.plse[((size_t)b * S + s) * a.HU + hu];
    }
    __syncthreads();

    for (int r = warp; r < R; r += kThreads / 32) {
        float *wr = w_s + r * S;
        float mx = -INFINITY;
        for (int s = lane; s < S; s += 32)
            mx = fmaxf(mx, wr[s]);
        for (int o = 16; o; o >>= 1)
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        float sum = 0.f;
        for (int s = lane; s < S; s += 32) {
            const float w = mx == -INFINITY ? 0.f : expf(wr[s] - mx);
            wr[s] = w;
            sum += w;
        }
        for (int o = 16; o; o >>= 1)
            sum += __shfl_xor_sync(0xffffffffu, sum, o);
        const float inv = sum > 0.f ? 1.f / sum : 0.f;
        for (int s = lane; s < S; s += 32)
            wr[s] *= inv;
        if (lane == 0 && a.lse && blockIdx.z == 0) {
            const int hu = a.mlra ? h * R + r : h;
            a.lse[(size_t)b * a.HU + hu] = (mx == -INFINITY || !(sum > 0.f)) ? -INFINITY : mx + logf(sum);
        }
    }
    __syncthreads();

    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    if (on) {
#pragma unroll
        for (int u = 0; u < PRE; ++u) {
            const int k = g + u * kGroups;
            const float w = k < rows ? w_s[k] : 0.f;
            acc.x = fmaf(w, v[u].x, acc.x);
            acc.y = fmaf(w, v[u].y, acc.y);
            acc.z = fmaf(w, v[u].z, acc.z);
            acc.w = fmaf(w, v[u].w, acc.w);
        }
        int k = g + PRE * kGroups;
        for (; k + 3 * kGroups < rows; k += 4 * kGroups) {
#pragma unroll
            for (int u = 0; u < 4; ++u)
                v[u] = __ldcs(row_ptr(k + u * kGroups));
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const float w = w_s[k + u * kGroups];
                acc.x = fmaf(w, v[u].x, acc.x);
                acc.y = fmaf(w, v[u].y, acc.y);
                acc.z = fmaf(w, v[u].z, acc.z);
                acc.w = fmaf(w, v[u].w, acc.w);
            }
        }
        for (; k < rows; k += kGroups) {
            const float4 x = __ldcs(row_ptr(k));
            const float w = w_s[k];
            acc.x = fmaf(w, x.x, acc.x);
            acc.y = fmaf(w, x.y, acc.y);
            acc.z = fmaf(w, x.z, acc.z);
            acc.w = fmaf(w, x.w, acc.w);
        }
    }
    acc_s[g * kV4 + q4] = acc;
    __syncthreads();
    if (tid < kV4 && on) {
        float4 sum = acc_s[tid];
        for (int gg = 1; gg < kGroups; ++gg) {
            const float4 x = acc_s[gg * kV4 + tid];
            sum.x += x.x;
            sum.y += x.y;
            sum.z += x.z;
            sum.w += x.w;
        }
        const size_t o = ((size_t)b * a.H + h) * a.Dv + col;
        if (a.out_fp32) {
            *reinterpret_cast<float4 *>(static_cast<float *>(a.out) + o) = sum;
        } else {
            const __nv_bfloat162 lo = __floats2bfloat162_rn(sum.x, sum.y);
            const __nv_bfloat162 hi = __floats2bfloat162_rn(sum.z, sum.w);
            uint2 packed;
            packed.x = *reinterpret_cast<const uint32_t *>(&lo);
            packed.y = *reinterpret_cast<const uint32_t *>(&hi);
            *reinterpret_cast<uint2 *>(static_cast<__nv_bfloat16 *>(a.out) + o) = packed;
        }
    }
}

}  // namespace

template <int PRE>
cudaError_t launch_combine_pre(const CombineArgs &a, size_t smem, cudaStream_t st)
{
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(combine_kernel<PRE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess)
            return e;
    }
    const int R = a.mlra ? a.NU : 1;
    const int cols = 4 * (kThreads / combine_groups(R * a.num_splits, a.Dv));
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(a.H, a.B, (a.Dv + cols - 1) / cols);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, combine_kernel<PRE>, a);
}

cudaError_t launch_combine(const CombineArgs &a, cudaStream_t st)
{
    const int R = a.mlra ? a.NU : 1;
    const int rows = R * a.num_splits;
    const size_t smem = (size_t)rows * sizeof(float);
    // rows one thread owns; the prefetch depth covers them, or most of them
    // (registers grow with it: depth 8 keeps eight blocks per SM, so the
    // usual grids stay resident in one wave)
    const int per = (rows + combine_groups(rows, a.Dv) - 1) / combine_groups(rows, a.Dv);
    if (per <= 2)
        return launch_combine_pre<2>(a, smem, st);
    if (per <= 4)
        return launch_combine_pre<4>(a, smem, st);
    if (per <= 10)
        return launch_combine_pre<8>(a, smem, st);
    return launch_combine_pre<16>(a, smem, st);
}

}  // namespace kvattn
