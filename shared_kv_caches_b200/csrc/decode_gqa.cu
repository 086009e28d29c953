// GQA decode: 4 query heads per KV head, head dim 128.
//
// A group of query heads shares one K/V head (MLRA page, GQA bullet), so one
// CTA owns (part s of the context, KV head, sequence b) and serves the 4 query
// heads of that KV head from one pass over its pages.
//
// Per CTA: one producer warp streams each 64-token page's K and V tiles of the
// KV head (2 x 16 KB) into a STAGES-deep shared-memory ring with 3-D TMA loads
// (128-byte swizzle, completion on an mbarrier); four consumer warps each own
// 16 tokens of every page and keep their own online-softmax state (running
// max m, sum l and output O per head, fp32, scores in base 2), so no
// CTA-wide barrier runs per page.  At the end of the part the four warp
// states are merged by their max (the same LSE merge the combine pass uses
// across parts) and the normalised part output and lse go to the workspace.
//
// The products run on the tensor cores as warp-level bf16 MMAs (m16n8k16,
// fp32 accumulate), transposed so that the warp's 16 tokens fill the MMA's 16
// rows and the 4 heads (padded to 8) its columns: S^T = K Q^T takes the K tile
// straight from shared memory (ldmatrix) with Q^T held in registers, and
// O^T = V^T P^T takes V through a transposing ldmatrix and P^T from the score
// fragments transposed in registers (movmatrix).  On the CUDA cores the bf16
// unpacking and the per-token reductions around the 16 384 FMAs per token
// cost more issue slots than the FMAs themselves.
#include <math.h>

#include "kvattn_internal.cuh"
#include "sm100.cuh"

namespace kvattn {

namespace {

constexpr int D = 128;
constexpr int G = 4;
constexpr int CW = 4;                        // consumer warps
constexpr int STAGES = 2;
constexpr int TPW = kPage / CW;              // tokens per warp per page
constexpr int THREADS = (CW + 1) * 32;
constexpr int BOX_BYTES = kPage * 64 * 2;    // 64 tokens x 64 dims (one 128-byte swizzle span)
constexpr int TILE_BYTES = 2 * BOX_BYTES;    // 64 tokens x 128 dims
constexpr int STAGE_BYTES = 2 * TILE_BYTES;  // K and V
constexpr float kLn2 = 0.69314718055994531f;

struct GqaSmem {
    unsigned char tiles[STAGES][STAGE_BYTES];   // 1024-byte aligned (swizzle atoms)
    float ow[CW][G][D];                         // per-warp outputs for the final merge
    float mw[CW][G];
    float lw[CW][G];
    uint64_t full[2 * STAGES];                  // one per slot (tied pages: two slots per stage)
    uint64_t empty[2 * STAGES];
    int skip[2 * STAGES];
    int last;
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

// c (16 x 8, fp32) += a (16 x 16, bf16, row) * b (16 x 8, bf16, col)
__device__ __forceinline__ void mma_bf16(float *c, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                         uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Transpose an 8 x 8 bf16 matrix held one fragment row pair per thread.
__device__ __forceinline__ uint32_t movm_t(uint32_t x)
{
    uint32_t y;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
    return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi)
{
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&v);
}

// TIED: one plane per page that serves as key and value (GTA)
template <bool TIED>
__global__ void __launch_bounds__(THREADS, 3) gqa_decode_kernel(const __grid_constant__ CUtensorMap kv_map,
                                                             const DecodeArgs a)
{
    extern __shared__ unsigned char smem_raw[];
    GqaSmem &S = *reinterpret_cast<GqaSmem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;

    const int L = row_context(a, b, threadIdx.x == 0 && split == 0 && kvh == 0);
    const int npages = (L + kPage - 1) / kPage;
    const int p0 = split * a.pages_per_split;
    const int n = max(0, min(npages, p0 + a.pages_per_split) - p0);

    // tied keys and values (GTA) fill half a stage per page: the ring then
    // holds twice as many one-tile slots, so as many bytes stay in flight
    constexpr bool tied = TIED;
    constexpr int nslots = tied ? 2 * STAGES : STAGES;
    constexpr int slot_bytes = tied ? TILE_BYTES : STAGE_BYTES;
    unsigned char *const ring = &S.tiles[0][0];

    if (threadIdx.x == 0) {
        for (int st = 0; st < nslots; ++st) {
            mbar_init(&S.full[st], 1);
            mbar_init(&S.empty[st], CW);
        }
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == CW) {
        // ------------------------------------------------------------ producer
        if (lane == 0 && n > 0) {
            prefetch_tmap(&kv_map);
            for (int i = 0; i < n; ++i) {
                const int st = i % nslots;
                if (i >= nslots && !mbar_wait(&S.empty[st], ((i / nslots) - 1) & 1)) {
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
                // tied: one tile serves as key and value
                mbar_arrive_expect_tx(&S.full[st], tied ? TILE_BYTES : STAGE_BYTES);
                const int zk = (int)(page * a.kv_planes * kPage), zv = zk + kPage;
                unsigned char *t = ring + (size_t)st * slot_bytes;
                tma_load_3d(t, &kv_map, 0, kvh, zk, &S.full[st]);
                tma_load_3d(t + BOX_BYTES, &kv_map, 64, kvh, zk, &S.full[st]);
                if (!tied) {
                    tma_load_3d(t + TILE_BYTES, &kv_map, 0, kvh, zv, &S.full[st]);
                    tma_load_3d(t + TILE_BYTES + BOX_BYTES, &kv_map, 64, kvh, zv, &S.full[st]);
                }
            }
        }
        return;
    }

    // ---------------------------------------------------------------- consumers
    // fragment coordinates: r = row group (token of S^T, dim of O^T, head of
    // the B operands), c = column pair (heads 2c, 2c+1 of S^T and O^T; only
    // c < 2 are real heads)
    const int r = lane >> 2, c = lane & 3;
    const int mrow = lane & 7, mat = lane >> 3;
    // Q^T as the B operand of S^T = K Q^T: b0 = dims 16kk + 2c.., b1 = + 8, head r
    uint32_t qb[D / 16][2];
    {
        const __nv_bfloat16 *qr = a.q_nope + ((size_t)b * a.H + kvh * G + (r < G ? r : 0)) * D;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
            qb[kk][0] = r < G ? *reinterpret_cast<const uint32_t *>(qr + 16 * kk + 2 * c) : 0u;
            qb[kk][1] = r < G ? *reinterpret_cast<const uint32_t *>(qr + 16 * kk + 8 + 2 * c) : 0u;
        }
    }
    float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};   // heads 2c, 2c+1
    float o[D / 16][4];                                                 // O^T: dims x heads
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt)
        o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;

    const int t0 = warp * TPW;
    for (int i = 0; i < n; ++i) {
        const int st = i % nslots;
        if (!mbar_wait(&S.full[st], (i / nslots) & 1)) {
            if (lane == 0)
                raise_error(a.err, KVATTN_DEVERR_WAIT_TIMEOUT);
            break;
        }
        const int ntok = min(kPage, L - (p0 + i) * kPage);
        const int nw = S.skip[st] ? 0 : min(max(ntok - t0, 0), TPW);
        if (nw > 0) {
            unsigned char *Kb = ring + (size_t)st * slot_bytes;
            unsigned char *Vb = tied ? Kb : Kb + TILE_BYTES;
            if (nw < TPW) {
                // value rows of this warp past the context: 0 * NaN would poison the MMA
                for (int idx = lane; idx < (TPW - nw) * (D / 8); idx += 32)
                    *reinterpret_cast<uint4 *>(Vb + chunk_off(t0 + nw + idx / (D / 8), idx % (D / 8))) =
                        make_uint4(0, 0, 0, 0);
                __syncwarp();
            }
            const uint32_t kbase = smem_u32(Kb), vbase = smem_u32(Vb);
            // S^T (16 tokens x 8 head columns) = K Q^T
            float s[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                uint32_t a0, a1, a2, a3;
                ldsm_x4(kbase + chunk_off(t0 + ((mat & 1) << 3) + mrow, 2 * kk + (mat >> 1)), a0, a1, a2, a3);
                mma_bf16(s, a0, a1, a2, a3, qb[kk][0], qb[kk][1]);
            }
            // online softmax per head over the warp's tokens (rows r and r + 8)
            float mx[2];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int tok = r + ((e >> 1) << 3);
                s[e] = tok < nw ? s[e] * a.scale_log2 : -INFINITY;
            }
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                mx[hh] = fmaxf(s[hh], s[2 + hh]);
                mx[hh] = fmaxf(mx[hh], __shfl_xor_sync(0xffffffffu, mx[hh], 4));
                mx[hh] = fmaxf(mx[hh], __shfl_xor_sync(0xffffffffu, mx[hh], 8));
                mx[hh] = fmaxf(mx[hh], __shfl_xor_sync(0xffffffffu, mx[hh], 16));
            }
            float alpha[2], m_use[2];
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const float m_new = fmaxf(m_run[hh], mx[hh]);
                m_use[hh] = m_new == -INFINITY ? 0.f : m_new;
                alpha[hh] = exp2f(m_run[hh] - m_use[hh]);
                m_run[hh] = m_new;
            }
            float p[4];
#pragma unroll
            for (int e = 0; e < 4; ++e)
                p[e] = exp2f(s[e] - m_use[e & 1]);
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                float ps = p[hh] + p[2 + hh];
                ps += __shfl_xor_sync(0xffffffffu, ps, 4);
                ps += __shfl_xor_sync(0xffffffffu, ps, 8);
                ps += __shfl_xor_sync(0xffffffffu, ps, 16);
                l_run[hh] = l_run[hh] * alpha[hh] + ps;
            }
            // P^T as the B operand of O^T = V^T P^T: tokens 2c.. (b0) and 8 + 2c.. (b1) of head r
            const uint32_t pb0 = movm_t(pack_bf16(p[0], p[1]));
            const uint32_t pb1 = movm_t(pack_bf16(p[2], p[3]));
#pragma unroll
            for (int mt = 0; mt < D / 16; ++mt) {
                o[mt][0] *= alpha[0];
                o[mt][1] *= alpha[1];
                o[mt][2] *= alpha[0];
                o[mt][3] *= alpha[1];
                uint32_t a0, a1, a2, a3;
                ldsm_x4_t(vbase + chunk_off(t0 + ((mat >> 1) << 3) + mrow, 2 * mt + (mat & 1)), a0, a1, a2, a3);
                mma_bf16(o[mt], a0, a1, a2, a3, pb0, pb1);
            }
            if (nw < TPW)
                fence_proxy_async_smem();   // the zeroed rows are rewritten by the next TMA load
        }
        __syncwarp();
        if (lane == 0)
            mbar_arrive(&S.empty[st]);
    }

    // merge the four warps' states and write this part's result
    if (c < 2) {
        if (r == 0) {
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                S.mw[warp][2 * c + hh] = m_run[hh];
                S.lw[warp][2 * c + hh] = l_run[hh];
            }
        }
#pragma unroll
        for (int mt = 0; mt < D / 16; ++mt)
#pragma unroll
            for (int e = 0; e < 4; ++e)
                S.ow[warp][2 * c + (e & 1)][16 * mt + r + ((e >> 1) << 3)] = o[mt][e];
    }
    named_sync(1, CW * 32);

    const int tid = threadIdx.x;
    float *po = a.po + (((size_t)b * a.num_splits + split) * a.HU + (size_t)kvh * G) * D;
    for (int idx = tid; idx < G * D; idx += CW * 32) {
        const int h = idx / D, d = idx % D;
        float mx = -INFINITY;
#pragma unroll
        for (int w = 0; w < CW; ++w)
            mx = fmaxf(mx, S.mw[w][h]);
        float num = 0.f, den = 0.f;
        if (mx != -INFINITY) {
#pragma unroll
            for (int w = 0; w < CW; ++w) {
                const float e = exp2f(S.mw[w][h] - mx);
                num = fmaf(e, S.ow[w][h][d], num);
                den = fmaf(e, S.lw[w][h], den);
            }
        }
        po[(size_t)h * D + d] = den > 0.f ? num / den : 0.f;
        if (d == 0) {
            float *pl = a.plse + ((size_t)b * a.num_splits + split) * a.HU + (size_t)kvh * G;
            pl[h] = den > 0.f ? (mx + log2f(den)) * kLn2 : -INFINITY;
        }
    }

    // the last part of (b, kvh) to finish merges all parts (the stage ring is
    // free by now and serves as scratch for the merge weights)
    if (finish_part(a, b * a.NU + kvh, &S.last, tid, CW * 32, 1))
        merge_group(a, b, kvh * G, G, D, reinterpret_cast<float *>(S.tiles[0]), tid, CW * 32, 1);
}

}  // namespace

size_t gqa_smem_bytes() { return sizeof(GqaSmem) + 1024; }

bool gqa_supported(const Problem &pr)
{
    // the in-kernel merge keeps G * splits weights in the stage ring
    return !pr.latent && pr.dn == D && pr.HPU == G && pr.mpps > 0 &&
           (size_t)G * kMaxSplits * sizeof(float) <= sizeof(GqaSmem::tiles);
}

cudaError_t launch_gqa(const DecodeArgs &a, cudaStream_t st)
{
    CUtensorMap map;
    const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)a.NU, (cuuint64_t)a.num_pages * a.kv_planes * kPage};
    const cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)a.NU * D * 2};
    const cuuint32_t box[3] = {64, 1, (cuuint32_t)kPage};
    if (encode_tiled(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<__nv_bfloat16 *>(a.kv), dims, strides,
                     box, CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    const size_t smem = gqa_smem_bytes();
    auto kern = a.kv_planes == 1 ? gqa_decode_kernel<true> : gqa_decode_kernel<false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess)
        return e;
    kern<<<dim3(a.num_splits, a.NU, a.B), THREADS, smem, st>>>(map, a);
    return cudaGetLastError();
}

}  // namespace kvattn
