// GQA decode on CUDA cores: 4 query heads per KV head, head dim 128.
//
// A group of query heads shares one K/V head (MLRA page, GQA bullet), so one
// CTA owns (part s of the context, KV head, sequence b) and serves the 4 query
// heads of that KV head from one pass over its pages.  At 4 flop per cache
// byte the work is HBM-bound and stays on the CUDA cores.
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
// Scores: the 128-wide dot is split over 8 lanes (16 dims each, q held in
// registers), and the 8 partial sums of 4 heads are reduced with a
// transposing butterfly (3 shuffle steps leave every lane with one finished
// (token, head) score).  P.V: every lane owns 4 of the 128 value dims for all
// 4 heads.  Shared-memory reads of K rows (one 128-byte line per 8 lanes) and
// V rows (256 bytes per warp) are bank-conflict free under the swizzle.
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
    float pw[CW][TPW][G];                       // per-warp probabilities of the current page
    float aw[CW][G];                            // per-warp rescale factors of the current page
    float mw[CW][G];
    float lw[CW][G];
    uint64_t full[STAGES];
    uint64_t empty[STAGES];
    int skip[STAGES];
    int last;
};

__device__ __forceinline__ float lo16(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float hi16(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ float dot8(const float *q, uint4 k)
{
    float s = q[0] * lo16(k.x);
    s = fmaf(q[1], hi16(k.x), s);
    s = fmaf(q[2], lo16(k.y), s);
    s = fmaf(q[3], hi16(k.y), s);
    s = fmaf(q[4], lo16(k.z), s);
    s = fmaf(q[5], hi16(k.z), s);
    s = fmaf(q[6], lo16(k.w), s);
    s = fmaf(q[7], hi16(k.w), s);
    return s;
}

__device__ __forceinline__ void load_q8(float *dst, const __nv_bfloat16 *src)
{
    const uint4 w = *reinterpret_cast<const uint4 *>(src);
    dst[0] = lo16(w.x);
    dst[1] = hi16(w.x);
    dst[2] = lo16(w.y);
    dst[3] = hi16(w.y);
    dst[4] = lo16(w.z);
    dst[5] = hi16(w.z);
    dst[6] = lo16(w.w);
    dst[7] = hi16(w.w);
}

__global__ void __launch_bounds__(THREADS) gqa_decode_kernel(const __grid_constant__ CUtensorMap kv_map,
                                                             const DecodeArgs a)
{
    extern __shared__ unsigned char smem_raw[];
    GqaSmem &S = *reinterpret_cast<GqaSmem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;

    int L = a.seq_lens[b];
    if (L > a.max_seq_len) {
        if (threadIdx.x == 0 && split == 0 && kvh == 0)
            raise_error(a.err, KVATTN_DEVERR_SEQ_TOO_LONG);
        L = a.max_seq_len;
    }
    L = max(L, 0);
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
        // ------------------------------------------------------------ producer
        if (lane == 0 && n > 0) {
            prefetch_tmap(&kv_map);
            for (int i = 0; i < n; ++i) {
                const int st = i % STAGES;
                if (i >= STAGES && !mbar_wait(&S.empty[st], ((i / STAGES) - 1) & 1)) {
                    raise_error(a.err, KVATTN_DEVERR_WAIT_TIMEOUT);
                    break;
                }
                const int pi = p0 + i;
                const long long page = a.block_table ? (long long)a.block_table[(size_t)b * a.mpps + pi]
                                                     : (long long)b * a.mpps + pi;
                if (page < 0 || page >= a.num_pages) {
                    raise_error(a.err, KVATTN_DEVERR_PAGE_OUT_OF_RANGE);
                    S.skip[st] = 1;
                    mbar_arrive(&S.full[st]);
                    continue;
                }
                S.skip[st] = 0;
                mbar_arrive_expect_tx(&S.full[st], STAGE_BYTES);
                const int zk = (int)(page * 2 * kPage), zv = zk + kPage;
                unsigned char *t = S.tiles[st];
                tma_load_3d(t, &kv_map, 0, kvh, zk, &S.full[st]);
                tma_load_3d(t + BOX_BYTES, &kv_map, 64, kvh, zk, &S.full[st]);
                tma_load_3d(t + TILE_BYTES, &kv_map, 0, kvh, zv, &S.full[st]);
                tma_load_3d(t + TILE_BYTES + BOX_BYTES, &kv_map, 64, kvh, zv, &S.full[st]);
            }
        }
        return;
    }

    // ---------------------------------------------------------------- consumers
    const int g = lane >> 3, j = lane & 7;
    const int hh = ((lane >> 2) & 1) * 2 + ((lane >> 1) & 1);   // head whose score this lane ends with
    float q0[G][8], q1[G][8];
#pragma unroll
    for (int h = 0; h < G; ++h) {
        const __nv_bfloat16 *qr = a.q_nope + ((size_t)b * a.H + kvh * G + h) * D;
        load_q8(q0[h], qr + 8 * j);
        load_q8(q1[h], qr + 64 + 8 * j);
    }
    float m_run = -INFINITY, l_run = 0.f;
    float O[G][4];
#pragma unroll
    for (int h = 0; h < G; ++h)
        O[h][0] = O[h][1] = O[h][2] = O[h][3] = 0.f;

    const int t0 = warp * TPW;
    const int vbox = lane >> 4, vchunk = (lane & 15) >> 1, vhalf = lane & 1;
    for (int i = 0; i < n; ++i) {
        const int st = i % STAGES;
        if (!mbar_wait(&S.full[st], (i / STAGES) & 1)) {
            if (lane == 0)
                raise_error(a.err, KVATTN_DEVERR_WAIT_TIMEOUT);
            break;
        }
        const int ntok = min(kPage, L - (p0 + i) * kPage);
        const int nw = S.skip[st] ? 0 : min(max(ntok - t0, 0), TPW);
        if (nw > 0) {
            const unsigned char *Kb = S.tiles[st];
            const unsigned char *Vb = Kb + TILE_BYTES;
            float sc[TPW / 4];
#pragma unroll
            for (int it = 0; it < TPW / 4; ++it) {
                const int t = t0 + 4 * it + g;
                const int off = t * 128 + ((j ^ (t & 7)) << 4);
                const uint4 k0 = *reinterpret_cast<const uint4 *>(Kb + off);
                const uint4 k1 = *reinterpret_cast<const uint4 *>(Kb + BOX_BYTES + off);
                float part[G];
#pragma unroll
                for (int h = 0; h < G; ++h)
                    part[h] = dot8(q0[h], k0) + dot8(q1[h], k1);
                // transposing butterfly over the 8 lanes of this token
                const bool up4 = (lane >> 2) & 1;
                const float a0 = (up4 ? part[2] : part[0]) +
                                 __shfl_xor_sync(0xffffffffu, up4 ? part[0] : part[2], 4);
                const float a1 = (up4 ? part[3] : part[1]) +
                                 __shfl_xor_sync(0xffffffffu, up4 ? part[1] : part[3], 4);
                const bool up2 = (lane >> 1) & 1;
                float c = (up2 ? a1 : a0) + __shfl_xor_sync(0xffffffffu, up2 ? a0 : a1, 2);
                c += __shfl_xor_sync(0xffffffffu, c, 1);
                sc[it] = (4 * it + g) < nw ? c * a.scale_log2 : -INFINITY;
            }
            // online softmax over this warp's tokens, per head hh
            float mt = sc[0];
#pragma unroll
            for (int it = 1; it < TPW / 4; ++it)
                mt = fmaxf(mt, sc[it]);
            mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 8));
            mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 16));
            const float m_new = fmaxf(m_run, mt);
            const float m_use = m_new == -INFINITY ? 0.f : m_new;
            const float alpha = exp2f(m_run - m_use);
            float ps = 0.f;
#pragma unroll
            for (int it = 0; it < TPW / 4; ++it) {
                sc[it] = exp2f(sc[it] - m_use);
                ps += sc[it];
            }
            ps += __shfl_xor_sync(0xffffffffu, ps, 8);
            ps += __shfl_xor_sync(0xffffffffu, ps, 16);
            l_run = l_run * alpha + ps;
            m_run = m_new;
            if ((lane & 1) == 0) {
#pragma unroll
                for (int it = 0; it < TPW / 4; ++it)
                    S.pw[warp][4 * it + g][hh] = sc[it];
                if (lane < 8)
                    S.aw[warp][hh] = alpha;
            }
            __syncwarp();

            // O = O * alpha + sum_t p_t v_t over this warp's tokens
            const float4 al = *reinterpret_cast<const float4 *>(S.aw[warp]);
            const float alv[G] = {al.x, al.y, al.z, al.w};
#pragma unroll
            for (int h = 0; h < G; ++h)
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    O[h][k] *= alv[h];
            const unsigned char *vrow = Vb + vbox * BOX_BYTES + vhalf * 8;
            for (int tl = 0; tl < nw; ++tl) {
                const int t = t0 + tl;
                const uint2 v = *reinterpret_cast<const uint2 *>(vrow + t * 128 + ((vchunk ^ (t & 7)) << 4));
                const float4 p4 = *reinterpret_cast<const float4 *>(S.pw[warp][tl]);
                const float vv[4] = {lo16(v.x), hi16(v.x), lo16(v.y), hi16(v.y)};
                const float pp[G] = {p4.x, p4.y, p4.z, p4.w};
#pragma unroll
                for (int h = 0; h < G; ++h)
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        O[h][k] = fmaf(pp[h], vv[k], O[h][k]);
            }
        }
        __syncwarp();
        if (lane == 0)
            mbar_arrive(&S.empty[st]);
    }

    // merge the four warps' states and write this part's result
    if ((lane & 1) == 0 && lane < 8) {
        S.mw[warp][hh] = m_run;
        S.lw[warp][hh] = l_run;
    }
#pragma unroll
    for (int h = 0; h < G; ++h)
        *reinterpret_cast<float4 *>(&S.ow[warp][h][4 * lane]) = make_float4(O[h][0], O[h][1], O[h][2], O[h][3]);
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
    const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)a.NU, (cuuint64_t)a.num_pages * 2 * kPage};
    const cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)a.NU * D * 2};
    const cuuint32_t box[3] = {64, 1, (cuuint32_t)kPage};
    if (encode_tiled(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<__nv_bfloat16 *>(a.kv), dims, strides,
                     box, CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    const size_t smem = gqa_smem_bytes();
    cudaError_t e = cudaFuncSetAttribute(gqa_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess)
        return e;
    gqa_decode_kernel<<<dim3(a.num_splits, a.NU, a.B), THREADS, smem, st>>>(map, a);
    return cudaGetLastError();
}

}  // namespace kvattn
