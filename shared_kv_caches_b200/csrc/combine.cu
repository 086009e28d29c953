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

constexpr int kThreads = 512;

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
    extern __shared__ float smem[];    // [R][S] merge weights, then [G][Dv] partial sums
    __shared__ float red[32];
    const int h = blockIdx.x, b = blockIdx.y;
    const int R = a.mlra ? a.NU : 1;
    const int S = a.num_splits;
    const int tid = threadIdx.x;
    float *w_s = smem;
    float *acc_s = smem + ((R * S + 3) & ~3);

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

    // G groups of Dv threads split the (branch, part) rows; each thread owns
    // one value column and keeps four row loads in flight (Dv <= 512)
    const int G = kThreads / a.Dv;
    const int g = tid / a.Dv, d = tid % a.Dv;
    const int rows = R * S;
    float acc = 0.f;
    if (g < G) {
        int k = g;
        for (; k + 3 * G < rows; k += 4 * G) {
            float v[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int kk = k + u * G, r = kk / S, s = kk % S;
                const int hu = a.mlra ? h * R + r : h;
                v[u] = a.po[(((size_t)b * S + s) * a.HU + hu) * a.Dv + d];
            }
#pragma unroll
            for (int u = 0; u < 4; ++u)
                acc = fmaf(w_s[k + u * G], v[u], acc);
        }
        for (; k < rows; k += G) {
            const int r = k / S, s = k % S;
            const int hu = a.mlra ? h * R + r : h;
            acc = fmaf(w_s[k], a.po[(((size_t)b * S + s) * a.HU + hu) * a.Dv + d], acc);
        }
        acc_s[g * a.Dv + d] = acc;
    }
    __syncthreads();
    if (tid < a.Dv) {
        float sum = 0.f;
        for (int gg = 0; gg < G; ++gg)
            sum += acc_s[gg * a.Dv + tid];
        const size_t o = ((size_t)b * a.H + h) * a.Dv + tid;
        if (a.out_fp32)
            static_cast<float *>(a.out)[o] = sum;
        else
            static_cast<__nv_bfloat16 *>(a.out)[o] = __float2bfloat16_rn(sum);
    }
}

}  // namespace

cudaError_t launch_combine(const CombineArgs &a, cudaStream_t st)
{
    const int R = a.mlra ? a.NU : 1;
    const int G = kThreads / a.Dv;
    const size_t smem = ((size_t)((R * a.num_splits + 3) & ~3) + (size_t)G * a.Dv) * sizeof(float);
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
