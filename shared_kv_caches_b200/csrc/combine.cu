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

__device__ float block_max(float v, float *red)
{
    for (int o = 16; o; o >>= 1)
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __syncthreads();
    if (lane == 0)
        red[w] = v;
    __syncthreads();
    float r = -INFINITY;
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i)
        r = fmaxf(r, red[i]);
    return r;
}

__device__ float block_sum(float v, float *red)
{
    for (int o = 16; o; o >>= 1)
        v += __shfl_xor_sync(0xffffffffu, v, o);
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __syncthreads();
    if (lane == 0)
        red[w] = v;
    __syncthreads();
    float r = 0.f;
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i)
        r += red[i];
    return r;
}

__global__ void __launch_bounds__(kThreads) combine_kernel(const CombineArgs a)
{
    extern __shared__ float w_s[];     // [R][S] merge weights
    __shared__ float red[32];
    const int h = blockIdx.x, b = blockIdx.y;
    const int R = a.mlra ? a.NU : 1;
    const int S = a.num_splits;
    const int tid = threadIdx.x;

    for (int r = 0; r < R; ++r) {
        const int hu = a.mlra ? h * R + r : h;
        const float *pl = a.plse + (size_t)b * S * a.HU + hu;
        float mx = -INFINITY;
        for (int s = tid; s < S; s += kThreads)
            mx = fmaxf(mx, pl[(size_t)s * a.HU]);
        mx = block_max(mx, red);
        float sum = 0.f;
        for (int s = tid; s < S; s += kThreads) {
            const float w = mx == -INFINITY ? 0.f : expf(pl[(size_t)s * a.HU] - mx);
            w_s[r * S + s] = w;
            sum += w;
        }
        sum = block_sum(sum, red);
        const float inv = sum > 0.f ? 1.f / sum : 0.f;
        for (int s = tid; s < S; s += kThreads)
            w_s[r * S + s] *= inv;
        if (tid == 0 && a.lse)
            a.lse[(size_t)b * a.HU + hu] = (mx == -INFINITY || !(sum > 0.f)) ? -INFINITY : mx + logf(sum);
    }
    __syncthreads();

    for (int d = tid; d < a.Dv; d += kThreads) {
        float acc = 0.f;
        for (int r = 0; r < R; ++r) {
            const int hu = a.mlra ? h * R + r : h;
            const float *po = a.po + ((size_t)b * S * a.HU + hu) * a.Dv + d;
            for (int s = 0; s < S; ++s) {
                const float w = w_s[r * S + s];
                if (w != 0.f)
                    acc = fmaf(w, po[(size_t)s * a.HU * a.Dv], acc);
            }
        }
        const size_t o = ((size_t)b * a.H + h) * a.Dv + d;
        if (a.out_fp32)
            static_cast<float *>(a.out)[o] = acc;
        else
            static_cast<__nv_bfloat16 *>(a.out)[o] = __float2bfloat16_rn(acc);
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
    combine_kernel<<<dim3(a.H, a.B), kThreads, smem, st>>>(a);
    return cudaGetLastError();
}

}  // namespace kvattn
