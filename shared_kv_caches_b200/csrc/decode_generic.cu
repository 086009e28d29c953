// Generic split-KV decode kernel on CUDA cores (every variant, any supported
// shape).  It is the correctness baseline of the library and the path for
// shapes the specialised kernels do not cover.
//
// One CTA owns (part s of the context, unit u, chunk of HC query heads,
// sequence b).  A unit is what a group of query heads attends: a KV head
// (GQA/MQA), the latent (MLA), latent group g (GLA) or latent branch r (MLRA).
// For each 64-token page of its part the CTA copies the unit's key columns
// (latent slice + shared rope key, or K and V rows) into shared memory, forms
// the base-2 scores of its heads, updates a running max / sum per head (online
// softmax in fp32) and accumulates p * v.  The part's normalised output and
// lse go to the workspace; the combine kernel merges the parts.
//
// MLA explainer (mlqm.cn/news/371735) section 2.3 gives the per-head formula,
// section 2.2 the key concatenation; the MLRA page (aitntnews.com
// newId=23265) the absorbed form and the per-branch attention; the GLA page
// (jsbsmhs.com/zixun/902167) the latent group a head reads.
#include <math.h>

#include "kvattn_internal.cuh"

namespace kvattn {

namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// bf16 elements per shared-memory row: the row's 32-bit word count is made odd
// so that 32 lanes reading the same column of 32 rows hit 32 banks.
__host__ __device__ inline int padded_stride(int d) { return ((d / 2) % 2 == 0) ? d + 2 : d; }

template <int HC>
__global__ void __launch_bounds__(kThreads) generic_decode_kernel(const DecodeArgs a)
{
    extern __shared__ __align__(16) unsigned char smem[];
    const int tid = threadIdx.x;
    pdl_launch_dependents();
    const int s = blockIdx.x;
    const int u = blockIdx.y / a.head_chunks;
    const int hc = blockIdx.y % a.head_chunks;
    const int b = blockIdx.z;
    const int Dk = a.dn + a.dr;
    const int Dv = a.dn;
    const int KS = padded_stride(Dk);
    const int VS = padded_stride(Dv);

    float *qs = reinterpret_cast<float *>(smem);          // [HC][Dk]
    float *sc = qs + HC * Dk;                              // [HC][64] scores, then weights
    float *m_s = sc + HC * kPage;                          // running max (base 2)
    float *l_s = m_s + HC;                                 // running sum
    float *al_s = l_s + HC;                                // rescale factor of this tile
    uint32_t *ks = reinterpret_cast<uint32_t *>(smem + ((HC * Dk + HC * kPage + 3 * HC) * 4 + 15) / 16 * 16);
    uint32_t *vs = ks + kPage * KS / 2;                    // GQA/MQA value rows

    const int L = row_context(a, b, tid == 0 && blockIdx.x == 0 && blockIdx.y == 0);
    const int npages = (L + kPage - 1) / kPage;
    const int p0 = s * a.pages_per_split;
    const int p1 = min(npages, p0 + a.pages_per_split);
    const int head0 = (a.mlra ? 0 : u * a.HPU) + hc * HC;

    float *po = a.po + ((size_t)b * a.num_splits + s) * a.HU * Dv;
    float *pl = a.plse + ((size_t)b * a.num_splits + s) * a.HU;

    // P.V mapping: thread owns value column pair cp for heads hgi, hgi+hg, ...
    const int NP = Dv / 2;
    const int hg = max(1, kThreads / NP);
    const int cp = tid % NP;
    const int hgi = tid / NP;
    const bool pv_on = hgi < hg && tid < NP * hg;

    float acc[HC][2];
#pragma unroll
    for (int k = 0; k < HC; ++k)
        acc[k][0] = acc[k][1] = 0.f;

    if (tid < HC) {
        m_s[tid] = -INFINITY;
        l_s[tid] = 0.f;
    }
    for (int idx = tid; idx < HC * Dk; idx += kThreads) {
        const int i = idx / Dk, d = idx % Dk;
        const int h = head0 + i;
        const size_t qrow = a.mlra ? ((size_t)(b * a.H + h) * a.NU + u) : (size_t)(b * a.H + h);
        const __nv_bfloat16 v = d < a.dn ? a.q_nope[qrow * a.dn + d] : a.q_rope[qrow * a.dr + (d - a.dn)];
        qs[idx] = __bfloat162float(v);
    }

    const int vec_k = Dk / 8;     // 16-byte vectors per key row
    const int vec_v = Dv / 8;
    for (int pi = p0; pi < p1; ++pi) {
        const long long page = row_page(a, b, pi);
        if (page < 0 || page >= a.num_pages) {
            if (tid == 0)
                raise_error(a.err, KVATTN_DEVERR_PAGE_OUT_OF_RANGE);
            continue;
        }
        const int ntok = min(kPage, L - pi * kPage);
        __syncthreads();   // previous tile fully consumed; q / stats initialised

        // stage the unit's key (and value) rows of this page
        for (int idx = tid; idx < ntok * vec_k; idx += kThreads) {
            const int t = idx / vec_k, v = idx % vec_k;
            const __nv_bfloat16 *src;
            if (a.latent) {
                const __nv_bfloat16 *row = a.kv + ((size_t)page * kPage + t) * a.row;
                src = v * 8 < a.dn ? row + (size_t)u * a.dn + v * 8 : row + (size_t)a.NU * a.dn + (v * 8 - a.dn);
            } else {
                src = a.kv + (((size_t)page * a.kv_planes + 0) * kPage + t) * a.row + (size_t)u * a.dn + v * 8;
            }
            const uint4 w = *reinterpret_cast<const uint4 *>(src);
            uint32_t *dst = ks + (t * KS) / 2 + v * 4;
            dst[0] = w.x;
            dst[1] = w.y;
            dst[2] = w.z;
            dst[3] = w.w;
        }
        if (!a.latent) {
            for (int idx = tid; idx < ntok * vec_v; idx += kThreads) {
                const int t = idx / vec_v, v = idx % vec_v;
                const __nv_bfloat16 *src =
                    a.kv + (((size_t)page * a.kv_planes + a.kv_planes - 1) * kPage + t) * a.row + (size_t)u * a.dn +
                    v * 8;
                const uint4 w = *reinterpret_cast<const uint4 *>(src);
                uint32_t *dst = vs + (t * VS) / 2 + v * 4;
                dst[0] = w.x;
                dst[1] = w.y;
                dst[2] = w.z;
                dst[3] = w.w;
            }
        }
        __syncthreads();

        // scores s[i][t] = scale * log2(e) * q_i . k_t
        {
            const int t = tid & (kPage - 1), hq = tid >> 6;
#pragma unroll
            for (int k = 0; k < (HC + 3) / 4; ++k) {
                const int i = hq + 4 * k;
                if (i < HC) {
                    float dot = 0.f;
                    if (t < ntok) {
                        const uint32_t *kr = ks + (t * KS) / 2;
                        const float2 *qr = reinterpret_cast<const float2 *>(qs + i * Dk);
                        for (int d2 = 0; d2 < Dk / 2; ++d2) {
                            const uint32_t w = kr[d2];
                            const float2 q2 = qr[d2];
                            dot = fmaf(q2.x, bf_lo(w), dot);
                            dot = fmaf(q2.y, bf_hi(w), dot);
                        }
                    }
                    sc[i * kPage + t] = t < ntok ? dot * a.scale_log2 : -INFINITY;
                }
            }
        }
        __syncthreads();

        // online softmax update, one warp per head
        {
            const int w = tid >> 5, lane = tid & 31;
            for (int i = w; i < HC; i += kThreads / 32) {
                const float v0 = sc[i * kPage + lane], v1 = sc[i * kPage + lane + 32];
                float mx = fmaxf(v0, v1);
#pragma unroll
                for (int o = 16; o; o >>= 1)
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
                const float m_old = m_s[i];
                const float m_new = fmaxf(m_old, mx);
                const float m_use = m_new == -INFINITY ? 0.f : m_new;
                const float e0 = exp2f(v0 - m_use), e1 = exp2f(v1 - m_use);
                sc[i * kPage + lane] = e0;
                sc[i * kPage + lane + 32] = e1;
                float sum = e0 + e1;
#pragma unroll
                for (int o = 16; o; o >>= 1)
                    sum += __shfl_xor_sync(0xffffffffu, sum, o);
                __syncwarp();
                if (lane == 0) {
                    const float al = exp2f(m_old - m_use);
                    al_s[i] = al;
                    l_s[i] = l_s[i] * al + sum;
                    m_s[i] = m_new;
                }
            }
        }
        __syncthreads();

        // acc = acc * alpha + sum_t p_t v_t
        if (pv_on) {
            const uint32_t *vb = a.latent ? ks : vs;
            const int vstride = (a.latent ? KS : VS) / 2;
#pragma unroll
            for (int k = 0; k < HC; ++k) {
                const int i = hgi + hg * k;
                if (i < HC) {
                    const float al = al_s[i];
                    acc[k][0] *= al;
                    acc[k][1] *= al;
                }
            }
            for (int t = 0; t < ntok; ++t) {
                const uint32_t w = vb[t * vstride + cp];
                const float v0 = bf_lo(w), v1 = bf_hi(w);
#pragma unroll
                for (int k = 0; k < HC; ++k) {
                    const int i = hgi + hg * k;
                    if (i < HC) {
                        const float p = sc[i * kPage + t];
                        acc[k][0] = fmaf(p, v0, acc[k][0]);
                        acc[k][1] = fmaf(p, v1, acc[k][1]);
                    }
                }
            }
        }
    }
    __syncthreads();

    if (pv_on) {
#pragma unroll
        for (int k = 0; k < HC; ++k) {
            const int i = hgi + hg * k;
            if (i < HC) {
                const int h = head0 + i;
                const int hu = a.mlra ? h * a.NU + u : h;
                const float l = l_s[i];
                const float inv = l > 0.f ? 1.f / l : 0.f;
                float2 o;
                o.x = acc[k][0] * inv;
                o.y = acc[k][1] * inv;
                *reinterpret_cast<float2 *>(po + (size_t)hu * Dv + 2 * cp) = o;
            }
        }
    }
    if (tid < HC) {
        const int h = head0 + tid;
        const int hu = a.mlra ? h * a.NU + u : h;
        const float l = l_s[tid];
        pl[hu] = l > 0.f ? (m_s[tid] + log2f(l)) * 0.69314718055994531f : -INFINITY;
    }
}

template <int HC>
cudaError_t launch_hc(const DecodeArgs &a, size_t smem, cudaStream_t st)
{
    cudaError_t e = cudaFuncSetAttribute(generic_decode_kernel<HC>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess)
        return e;
    dim3 grid(a.num_splits, a.NU * a.head_chunks, a.B);
    generic_decode_kernel<HC><<<grid, kThreads, smem, st>>>(a);
    return cudaGetLastError();
}

}  // namespace

size_t generic_smem_bytes(const Problem &pr, int HC)
{
    size_t head = ((size_t)HC * pr.Dk + (size_t)HC * kPage + 3 * (size_t)HC) * 4;
    head = (head + 15) / 16 * 16;
    size_t kbytes = (size_t)kPage * padded_stride(pr.Dk) * 2;
    size_t vbytes = pr.latent ? 0 : (size_t)kPage * padded_stride(pr.Dv) * 2;
    return head + kbytes + vbytes;
}

cudaError_t launch_generic(const DecodeArgs &a, int HC, cudaStream_t st)
{
    Problem pr{};
    pr.Dk = a.dn + a.dr;
    pr.Dv = a.dn;
    pr.latent = a.latent != 0;
    const size_t smem = generic_smem_bytes(pr, HC);
    switch (HC) {
    case 1: return launch_hc<1>(a, smem, st);
    case 2: return launch_hc<2>(a, smem, st);
    case 4: return launch_hc<4>(a, smem, st);
    case 8: return launch_hc<8>(a, smem, st);
    case 16: return launch_hc<16>(a, smem, st);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace kvattn
