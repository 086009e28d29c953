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

// One block per (head, sequence, chunk of value columns).  Warp 0 turns the
// parts' lse values into merge weights (per branch for MLRA; every block of a
// head recomputes them, which is cheap); then G groups of 128/G threads split
// the (branch, part) rows, each thread owning four value columns (float4)
// with four row loads in flight; the groups meet in shared memory.
__global__ void __launch_bounds__(kThreads) combine_kernel(const CombineArgs a)
{
    extern __shared__ float w_s[];     // [R][S] merge weights
    __shared__ float4 acc_s[kMaxV4];
    const int h = blockIdx.x, b = blockIdx.y;
    const int R0 = a.mlra ? a.NU : 1;
    const int kGroups = combine_groups(R0 * a.num_splits, a.Dv);
    const int kV4 = kThreads / kGroups;
    const int c0 = blockIdx.z * 4 * kV4;
    const int R = a.mlra ? a.NU : 1;
    const int S = a.num_splits;
    const int tid = threadIdx.x, lane = tid & 31;

    if (tid < 32) {
        for (int r = 0; r < R; ++r) {
            const int hu = a.mlra ? h * R + r : h;
            const float *pl = a.plse + (size_t)b * S * a.HU + hu;
            float mx = -INFINITY;
            for (int s = lane; s < S; s += 32)
                mx = fmaxf(mx, pl[(size_t)s * a.HU]);
            for (int o = 16; o; o >>= 1)
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            float sum = 0.f;
            for (int s = lane; s < S; s += 32) {
                const float w = mx == -INFINITY ? 0.f : expf(pl[(size_t)s * a.HU] - mx);
                w_s[r * S + s] = w;
                sum += w;
            }
            for (int o = 16; o; o >>= 1)
                sum += __shfl_xor_sync(0xffffffffu, sum, o);
            const float inv = sum > 0.f ? 1.f / sum : 0.f;
            for (int s = lane; s < S; s += 32)
                w_s[r * S + s] *= inv;
            if (lane == 0 && a.lse && blockIdx.z == 0)
                a.lse[(size_t)b * a.HU + hu] = (mx == -INFINITY || !(sum > 0.f)) ? -INFINITY : mx + logf(sum);
        }
    }
    __syncthreads();

    const int g = tid / kV4, q4 = tid % kV4;
    const int col = c0 + 4 * q4;
    const bool on = col < a.Dv;
    const int rows = R * S;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    if (on) {
        auto row_ptr = [&](int k) {
            const int r = k / S, s = k % S;
            const int hu = a.mlra ? h * R + r : h;
            return reinterpret_cast<const float4 *>(a.po + (((size_t)b * S + s) * a.HU + hu) * a.Dv + col);
        };
        int k = g;
        for (; k + 3 * kGroups < rows; k += 4 * kGroups) {
            float4 v[4];
#pragma unroll
            for (int u = 0; u < 4; ++u)
                v[u] = *row_ptr(k + u * kGroups);
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
            const float4 v = *row_ptr(k);
            const float w = w_s[k];
            acc.x = fmaf(w, v.x, acc.x);
            acc.y = fmaf(w, v.y, acc.y);
            acc.z = fmaf(w, v.z, acc.z);
            acc.w = fmaf(w, v.w, acc.w);
        }
    }
    acc_s[g * kV4 + q4] = acc;
    __syncthreads();
    if (tid < kV4 && on) {
        float4 sum = acc_s[tid];
        for (int gg = 1; gg < kGroups; ++gg) {
            const float4 v = acc_s[gg * kV4 + tid];
            sum.x += v.x;
            sum.y += v.y;
            sum.z += v.z;
            sum.w += v.w;
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

cudaError_t launch_combine(const CombineArgs &a, cudaStream_t st)
{
    const int R = a.mlra ? a.NU : 1;
    const size_t smem = (size_t)R * a.num_splits * sizeof(float);
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(combine_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess)
            return e;
    }
    const int cols = 4 * (kThreads / combine_groups(R * a.num_splits, a.Dv));
    combine_kernel<<<dim3(a.H, a.B, (a.Dv + cols - 1) / cols), kThreads, smem, st>>>(a);
    return cudaGetLastError();
}

}  // namespace kvattn
