// MQA decode with one wide KV head (the MFA page's single KV head at decode
// time): 32 query heads share K and V of head dim 256.
//
// At 32 flop per cache byte the scores and P.V no longer fit the CUDA cores
// at HBM speed, so both products run on the tensor cores with warp-level
// bf16 MMAs (m16n8k16, fp32 accumulate) whose operands come from shared
// memory through ldmatrix; the kernel stays HBM-bound.
//
// Per CTA (part s of the context, KV head, sequence b): one producer warp
// streams each 64-token page's K and V tiles (2 x 32 KB) into a STAGES-deep
// ring with 3-D TMA loads (128-byte swizzle).  Four consumer warps split the
// work as (16-head group) x (128-dim half of the value): each computes the
// 16 x 64 score tile of its heads (the two warps of a head group both do, so
// no scores cross warps), keeps the online-softmax state of its 16 rows in
// registers (fp32, base 2), turns the scores into the bf16 A operand of P.V
// in registers, and accumulates its 16 x 128 output slice.  Token slots past
// the context are masked in the scores and their value rows are zeroed in
// shared memory first, since 0 * NaN would still poison an MMA.
#include <math.h>

#include "kvattn_internal.cuh"
#include "sm100.cuh"

namespace kvattn {

namespace {

constexpr int D = 256;
constexpr int HEADS = 32;
constexpr int HG = HEADS / 16;               // 16-head groups
constexpr int VH = D / 128;                  // 128-dim value slices
constexpr int CW = HG * VH;                  // consumer warps
constexpr int THREADS = (CW + 1) * 32;
constexpr int STAGES = 3;
constexpr int BOX_BYTES = kPage * 64 * 2;    // 64 tokens x 64 dims
constexpr int TILE_BYTES = (D / 64) * BOX_BYTES;
constexpr int STAGE_BYTES = 2 * TILE_BYTES;
constexpr int KSTEPS = D / 16;
constexpr float kLn2 = 0.69314718055994531f;

struct MqaSmem {
    unsigned char tiles[STAGES][STAGE_BYTES];
    uint64_t full[STAGES];
    uint64_t empty[STAGES];
    int skip[STAGES];
};

// Byte offset of 16-byte chunk c (8 dims) of token row t in a swizzled tile.
__device__ __forceinline__ uint32_t chunk_off(int t, int c)
{
    return (uint32_t)((c >> 3) * BOX_BYTES + t * 128 + (((c & 7) ^ (t & 7)) << 4));
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

__device__ __forceinline__ void mma_bf16(float *c, const uint32_t *a, uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi)
{
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&v);
}

__global__ void __launch_bounds__(THREADS, 1) mqa_mma_decode_kernel(const __grid_constant__ CUtensorMap kv_map,
                                                                   const DecodeArgs a)
{
    extern __shared__ unsigned char smem_raw[];
    MqaSmem &S = *reinterpret_cast<MqaSmem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
    pdl_launch_dependents();

    const int L = row_context(a, b, threadIdx.x == 0 && split == 0 && kvh == 0);
    const int npages = (L + kPage - 1) / kPage;
    const int p0 = split * a.pages_per_split;
    const int n = max(0, min(npages, p0 + a.pages_per_split) - p0);

    if (threadIdx.x == 0) {
        for (int st = 0; st < STAGES; ++st) {
            mbar_init(&S.full[st], 1);
            mbar_init(&S.empty[st], CW);
        }
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == CW) {
        if (lane == 0 && n > 0) {
            prefetch_tmap(&kv_map);
            for (int i = 0; i < n; ++i) {
                const int st = i % STAGES;
                if (i >= STAGES && !mbar_wait(&S.empty[st], ((i / STAGES) - 1) & 1)) {
                    raise_error(a.err, KVATTN_DEVERR_WAIT_TIMEOUT);
                    break;
                }
                const int pi = p0 + i;
                const long long page = row_page(a, b, pi);
                if (page < 0 || page >= a.num_pages) {
                    raise_error(a.err, KVATTN_DEVERR_PAGE_OUT_OF_RANGE);
                    S.skip[st] = 1;
                    mbar_arrive(&S.full[st]);
                    continue;
                }
                S.skip[st] = 0;
                // tied keys and values (MFA-KR): one tile serves as both
                const bool tied = a.kv_planes == 1;
                mbar_arrive_expect_tx(&S.full[st], tied ? TILE_BYTES : STAGE_BYTES);
                const int zk = (int)(page * a.kv_planes * kPage), zv = zk + kPage;
                unsigned char *t = S.tiles[st];
#pragma unroll
                for (int x = 0; x < D / 64; ++x) {
                    tma_load_3d(t + x * BOX_BYTES, &kv_map, 64 * x, kvh, zk, &S.full[st]);
                    if (!tied)
                        tma_load_3d(t + TILE_BYTES + x * BOX_BYTES, &kv_map, 64 * x, kvh, zv, &S.full[st]);
                }
            }
        }
        return;
    }

    const int hg = warp % HG, vh = warp / HG;
    const int r = lane >> 2, c = lane & 3;
    const int head0 = kvh * HEADS + hg * 16;

    // Q fragments of this warp's 16 heads over the whole head dim (A operand)
    uint32_t qf[KSTEPS][4];
    {
        const __nv_bfloat16 *q0 = a.q_nope + ((size_t)b * a.H + head0 + r) * D;
        const __nv_bfloat16 *q8 = q0 + 8 * D;
#pragma unroll
        for (int kk = 0; kk < KSTEPS; ++kk) {
            qf[kk][0] = *reinterpret_cast<const uint32_t *>(q0 + 16 * kk + 2 * c);
            qf[kk][1] = *reinterpret_cast<const uint32_t *>(q8 + 16 * kk + 2 * c);
            qf[kk][2] = *reinterpret_cast<const uint32_t *>(q0 + 16 * kk + 8 + 2 * c);
            qf[kk][3] = *reinterpret_cast<const uint32_t *>(q8 + 16 * kk + 8 + 2 * c);
        }
    }
    float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
    float o[16][4];
#pragma unroll
    for (int nt = 0; nt < 16; ++nt)
        o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.f;

    const int mrow = lane & 7, mat = lane >> 3;
    for (int i = 0; i < n; ++i) {
        const int st = i % STAGES;
        if (!mbar_wait(&S.full[st], (i / STAGES) & 1)) {
            if (lane == 0)
                raise_error(a.err, KVATTN_DEVERR_WAIT_TIMEOUT);
            break;
        }
        const int ntok = S.skip[st] ? 0 : min(kPage, L - (p0 + i) * kPage);
        unsigned char *Kb = S.tiles[st];
        unsigned char *Vb = a.kv_planes == 1 ? Kb : Kb + TILE_BYTES;
        if (ntok > 0 && ntok < kPage) {
            // zero this warp's value slice of the slots past the context (the two
            // warps of a value half write the same zeros, then both wait)
            for (int idx = lane + 32 * hg; idx < (kPage - ntok) * 16; idx += 32 * HG) {
                const int t = ntok + idx / 16, cc = vh * 16 + (idx % 16);
                *reinterpret_cast<uint4 *>(Vb + chunk_off(t, cc)) = make_uint4(0, 0, 0, 0);
            }
            // the next TMA load into this stage (async proxy) must land after these stores
            fence_proxy_async_smem();
            named_sync(2 + vh, 32 * HG);
        }
        if (ntok > 0) {
            const uint32_t kbase = smem_u32(Kb), vbase = smem_u32(Vb);
            // S = Q K^T for 16 heads x 64 tokens
            float s[8][4];
#pragma unroll
            for (int nt = 0; nt < 8; ++nt)
                s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
#pragma unroll
            for (int kk = 0; kk < KSTEPS; ++kk) {
#pragma unroll
                for (int np = 0; np < 4; ++np) {
                    const int t = np * 16 + (mat >> 1) * 8 + mrow;
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4(kbase + chunk_off(t, 2 * kk + (mat & 1)), b0, b1, b2, b3);
                    mma_bf16(s[2 * np], qf[kk], b0, b1);
                    mma_bf16(s[2 * np + 1], qf[kk], b2, b3);
                }
            }
            // online softmax on rows r and r + 8
            float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
                const int t = nt * 8 + 2 * c;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int tt = t + (e & 1);
                    s[nt][e] = tt < ntok ? s[nt][e] * a.scale_log2 : -INFINITY;
                    mx[e >> 1] = fmaxf(mx[e >> 1], s[nt][e]);
                }
            }
            float alpha[2], m_use[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 1));
                mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 2));
                const float m_new = fmaxf(m_run[h], mx[h]);
                m_use[h] = m_new == -INFINITY ? 0.f : m_new;
                alpha[h] = exp2f(m_run[h] - m_use[h]);
                m_run[h] = m_new;
            }
            float ps[2] = {0.f, 0.f};
            uint32_t pf[4][4];
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    s[nt][e] = exp2f(s[nt][e] - m_use[e >> 1]);
                    ps[e >> 1] += s[nt][e];
                }
                const int kk = nt >> 1, hi = nt & 1;
                pf[kk][2 * hi + 0] = pack_bf16(s[nt][0], s[nt][1]);
                pf[kk][2 * hi + 1] = pack_bf16(s[nt][2], s[nt][3]);
            }
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                ps[h] += __shfl_xor_sync(0xffffffffu, ps[h], 1);
                ps[h] += __shfl_xor_sync(0xffffffffu, ps[h], 2);
                l_run[h] = l_run[h] * alpha[h] + ps[h];
            }
#pragma unroll
            for (int nt = 0; nt < 16; ++nt) {
                o[nt][0] *= alpha[0];
                o[nt][1] *= alpha[0];
                o[nt][2] *= alpha[1];
                o[nt][3] *= alpha[1];
            }
            // O += P V over this warp's 128 value dims
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const int t = kk * 16 + (mat & 1) * 8 + mrow;
#pragma unroll
                for (int np = 0; np < 8; ++np) {
                    const int cc = vh * 16 + np * 2 + (mat >> 1);
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4_t(vbase + chunk_off(t, cc), b0, b1, b2, b3);
                    mma_bf16(o[2 * np], pf[kk], b0, b1);
                    mma_bf16(o[2 * np + 1], pf[kk], b2, b3);
                }
            }
        }
        __syncwarp();
        if (lane == 0)
            mbar_arrive(&S.empty[st]);
    }

    // this warp's 16 heads x 128 dims of the part result
    const size_t rowbase = ((size_t)b * a.num_splits + split) * a.HU + head0;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const float inv = l_run[h] > 0.f ? 1.f / l_run[h] : 0.f;
        float *dst = a.po + (rowbase + r + 8 * h) * D + vh * 128;
#pragma unroll
        for (int nt = 0; nt < 16; ++nt)
            *reinterpret_cast<float2 *>(dst + nt * 8 + 2 * c) =
                make_float2(o[nt][2 * h] * inv, o[nt][2 * h + 1] * inv);
        if (vh == 0 && c == 0)
            a.plse[rowbase + r + 8 * h] = l_run[h] > 0.f ? (m_run[h] + log2f(l_run[h])) * kLn2 : -INFINITY;
    }
}

}  // namespace

bool mqa_mma_supported(const Problem &pr)
{
    return !pr.latent && pr.dn == D && pr.HPU == HEADS;
}

cudaError_t launch_mqa_mma(const DecodeArgs &a, cudaStream_t st)
{
    CUtensorMap map;
    const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)a.NU, (cuuint64_t)a.num_pages * a.kv_planes * kPage};
    const cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)a.NU * D * 2};
    const cuuint32_t box[3] = {64, 1, (cuuint32_t)kPage};
    if (encode_tiled(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<__nv_bfloat16 *>(a.kv), dims, strides,
                     box, CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    const size_t smem = sizeof(MqaSmem) + 1024;
    cudaError_t e =
        cudaFuncSetAttribute(mqa_mma_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess)
        return e;
    mqa_mma_decode_kernel<<<dim3(a.num_splits, a.NU, a.B), THREADS, smem, st>>>(map, a);
    return cudaGetLastError();
}

}  // namespace kvattn
