// GQA decode over an fp8 (e4m3) KV cache: 4 query heads per KV head, head
// dim 128.
//
// The cache holds each K and V element as one e4m3 byte with one scale per
// tensor (k_scale, v_scale): the key is k_scale * K8, the value v_scale * V8.
// Halving the bytes per token halves the HBM traffic of this HBM-bound decode
// (GTA/GLA page, "Mamba核心作者新作…": the largest-model serving test runs in
// FP8; MFA page, "突破大模型推理瓶颈…", closing paragraph: quantisation is the
// planned next step; neither fixes the format: e4m3 with per-tensor scales).  Scores are k_scale * (q . K8): the scale joins the
// softmax scale; outputs are v_scale * sum_j p_j V8_j: the scale multiplies
// the normalised part output.
//
// A producer warp streams each page's K and V tiles (64 tokens x 128 bytes
// each, one TMA box with the 128-byte swizzle) into a four-stage ring (the
// byte tiles are half the size of bf16 ones, so twice the stages keep as
// many bytes in flight); four consumer warps each own 16 tokens of a page.
// Each lane loads its bytes of the warp's K and V rows straight into
// registers (16-byte loads, conflict-free under the swizzle), the warp
// releases the stage at once, and the bytes become the f16 fragments of the
// transposed warp-level MMAs in registers (cvt.rn.f16x2.e4m3x2: e4m3 values
// are exactly representable in f16):
//  - S^T = K Q^T contracts over the head dims, so the dims may take any
//    order that K and Q share: step kk = 4s + w of lane (r, c) holds dims
//    32c + 16s + 4w .. +3, which is the 16-byte chunk 2c + s of rows r and
//    r + 8, read whole;
//  - O^T = V^T P^T contracts over tokens and its rows are output dims: lane
//    (r, c) reads chunk r (dims 16r .. 16r + 15) of its four tokens 2c, 2c+1,
//    8+2c, 9+2c and pairs the tokens byte by byte (prmt); row r of M-tile mt
//    is then dim 16r + 4(mt/2) + 2(mt%2), row r + 8 the next dim.
// The query (bf16) is used as f16, loaded once in the dims' order.  The last
// CTA of each (sequence, KV head) merges the parts.
#include <math.h>

#include <cuda_fp16.h>

#include "kvattn_internal.cuh"
#include "sm100.cuh"

namespace kvattn {

namespace {

constexpr int D = 128;
constexpr int G = 4;
constexpr int CW = 4;                        // consumer warps
constexpr int STAGES = 4;
constexpr int TPW = kPage / CW;              // tokens per warp per page
constexpr int THREADS = (CW + 1) * 32;
constexpr int TILE8 = kPage * D;             // fp8 K (or V) tile: 64 tokens x 128 bytes, one swizzle span
constexpr int STAGE8 = 2 * TILE8;            // K and V
constexpr float kLn2 = 0.69314718055994531f;

struct Fp8Smem {
    unsigned char tiles[STAGES][STAGE8];        // fp8 stages (1024-byte aligned, swizzle atoms)
    float ow[CW][G][D];                         // per-warp outputs for the final merge
    float mw[CW][G];
    float lw[CW][G];
    uint64_t full[STAGES];
    uint64_t empty[STAGES];
    int skip[STAGES];
    int last;
};

// Word i (compile-time after unrolling) of a 16-byte load.
__device__ __forceinline__ uint32_t word_of(const uint4 &v, int i)
{
    return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

// Two e4m3 bytes (low byte first) to two f16 (low half first), exactly.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t v)
{
    uint32_t r;
    const uint16_t h = (uint16_t)(v & 0xffffu);
    asm("{\n\t.reg .b16 t;\n\tmov.b16 t, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, t;\n\t}" : "=r"(r) : "h"(h));
    return r;
}

// c (16 x 8, fp32) += a (16 x 16, f16, row) * b (16 x 8, f16, col)
__device__ __forceinline__ void mma_f16(float *c, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                        uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Transpose an 8 x 8 16-bit matrix held one fragment row pair per thread.
__device__ __forceinline__ uint32_t movm_t(uint32_t x)
{
    uint32_t y;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
    return y;
}

__device__ __forceinline__ uint32_t pack_f16(float lo, float hi)
{
    const __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&v);
}

// A pair of bf16 (as loaded from the query) to a pair of f16.
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t v)
{
    const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162 *>(&v);
    const float2 f = __bfloat1622float2(b);
    return pack_f16(f.x, f.y);
}

__global__ void __launch_bounds__(THREADS, 3) gqa_fp8_decode_kernel(const __grid_constant__ CUtensorMap kv_map,
                                                                 const DecodeArgs a, float kscale_log2, float v_scale)
{
    extern __shared__ unsigned char smem_raw[];
    Fp8Smem &S = *reinterpret_cast<Fp8Smem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;

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
                const long long page = row_page(a, b, pi);
                if (page < 0 || page >= a.num_pages) {
                    raise_error(a.err, KVATTN_DEVERR_PAGE_OUT_OF_RANGE);
                    S.skip[st] = 1;
                    mbar_arrive(&S.full[st]);
                    continue;
                }
                S.skip[st] = 0;
                mbar_arrive_expect_tx(&S.full[st], STAGE8);
                const int zk = (int)(page * 2 * kPage), zv = zk + kPage;
                unsigned char *t = S.tiles[st];
                tma_load_3d(t, &kv_map, 0, kvh, zk, &S.full[st]);
                tma_load_3d(t + TILE8, &kv_map, 0, kvh, zv, &S.full[st]);
            }
        }
        return;
    }

    // ---------------------------------------------------------------- consumers
    // fragment coordinates: r = row group (token of S^T, dims of O^T, head of
    // the B operands), c = column pair (heads 2c, 2c+1 of S^T and O^T; only
    // c < 2 are real heads)
    const int r = lane >> 2, c = lane & 3;
    // Q^T as the B operand of S^T = K Q^T (head r) in the dims' order of the
    // K fragments: step kk = 4s + w holds dims 32c + 16s + 4w + {0, 1} (b0)
    // and + {2, 3} (b1)
    uint32_t qb[D / 16][2];
    {
        const __nv_bfloat16 *qr = a.q_nope + ((size_t)b * a.H + kvh * G + (r < G ? r : 0)) * D + 32 * c;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
            const int d = 16 * (kk >> 2) + 4 * (kk & 3);
            qb[kk][0] = r < G ? bf16x2_to_f16x2(*reinterpret_cast<const uint32_t *>(qr + d)) : 0u;
            qb[kk][1] = r < G ? bf16x2_to_f16x2(*reinterpret_cast<const uint32_t *>(qr + d + 2)) : 0u;
        }
    }
    float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};   // heads 2c, 2c+1
    float o[D / 16][4];                                                 // O^T: dims x heads
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt)
        o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;

    const int t0 = warp * TPW;
    for (int i = 0; i < n; ++i) {
        const int st = i % STAGES;
        if (!mbar_wait(&S.full[st], (i / STAGES) & 1)) {
            if (lane == 0)
                raise_error(a.err, KVATTN_DEVERR_WAIT_TIMEOUT);
            break;
        }
        const int ntok = min(kPage, L - (p0 + i) * kPage);
        const int nw = S.skip[st] ? 0 : min(max(ntok - t0, 0), TPW);
        // this lane's bytes of the warp's rows: row t of a tile sits at t * 128
        // with its 16-byte chunk j at (j ^ (t & 7)) * 16; t0 is a multiple of 8
        uint4 kr[2][2], vr[4];
        if (nw > 0) {
            const unsigned char *kt = S.tiles[st] + t0 * 128, *vt = kt + TILE8;
            // K: chunk 2c + s of rows r and r + 8
#pragma unroll
            for (int s2 = 0; s2 < 2; ++s2) {
                const int off = ((2 * c + s2) ^ r) << 4;
                kr[s2][0] = *reinterpret_cast<const uint4 *>(kt + r * 128 + off);
                kr[s2][1] = *reinterpret_cast<const uint4 *>(kt + (r + 8) * 128 + off);
            }
            // V: chunk r of tokens 2c, 2c + 1, 8 + 2c, 9 + 2c; tokens past the
            // context become zeros (0 * NaN would poison the MMA)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int t = 2 * c + (j & 1) + ((j >> 1) << 3);
                vr[j] = t < nw ? *reinterpret_cast<const uint4 *>(vt + t * 128 + ((r ^ (t & 7)) << 4))
                               : make_uint4(0u, 0u, 0u, 0u);
            }
        }
        // the stage is free for the next TMA load once every lane holds its bytes
        __syncwarp();
        if (lane == 0)
            mbar_arrive(&S.empty[st]);
        if (nw > 0) {
            // S^T (16 tokens x 8 head columns) = K Q^T; a0/a2 = row r, a1/a3 =
            // row r + 8, low/high byte pair of one word = dims + {0, 1} / + {2, 3}
            float s[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t w0 = word_of(kr[kk >> 2][0], kk & 3), w1 = word_of(kr[kk >> 2][1], kk & 3);
                mma_f16(s, e4m3x2_to_f16x2(w0), e4m3x2_to_f16x2(w1), e4m3x2_to_f16x2(w0 >> 16),
                        e4m3x2_to_f16x2(w1 >> 16), qb[kk][0], qb[kk][1]);
            }
            // online softmax per head over the warp's tokens (rows r and r + 8)
            float mx[2];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int tok = r + ((e >> 1) << 3);
                s[e] = tok < nw ? s[e] * kscale_log2 : -INFINITY;
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
            const uint32_t pb0 = movm_t(pack_f16(p[0], p[1]));
            const uint32_t pb1 = movm_t(pack_f16(p[2], p[3]));
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                // byte pairs of tokens (2c, 2c + 1) and (8 + 2c, 9 + 2c), dims 16r + 4w .. + 3
                const uint32_t x0 = word_of(vr[0], w), x1 = word_of(vr[1], w);
                const uint32_t x2 = word_of(vr[2], w), x3 = word_of(vr[3], w);
                const uint32_t lo01 = __byte_perm(x0, x1, 0x5140), hi01 = __byte_perm(x0, x1, 0x7362);
                const uint32_t lo23 = __byte_perm(x2, x3, 0x5140), hi23 = __byte_perm(x2, x3, 0x7362);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    o[2 * w][e] *= alpha[e & 1];
                    o[2 * w + 1][e] *= alpha[e & 1];
                }
                // M-tile 2w: rows r / r + 8 = dims 16r + 4w / + 1; M-tile 2w + 1: + 2 / + 3
                mma_f16(o[2 * w], e4m3x2_to_f16x2(lo01), e4m3x2_to_f16x2(lo01 >> 16), e4m3x2_to_f16x2(lo23),
                        e4m3x2_to_f16x2(lo23 >> 16), pb0, pb1);
                mma_f16(o[2 * w + 1], e4m3x2_to_f16x2(hi01), e4m3x2_to_f16x2(hi01 >> 16), e4m3x2_to_f16x2(hi23),
                        e4m3x2_to_f16x2(hi23 >> 16), pb0, pb1);
            }
        }
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
        for (int mt = 0; mt < D / 16; ++mt) {
            const int d0 = 16 * r + 4 * (mt >> 1) + 2 * (mt & 1);
#pragma unroll
            for (int e = 0; e < 4; ++e)
                S.ow[warp][2 * c + (e & 1)][d0 + (e >> 1)] = o[mt][e];
        }
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
        po[(size_t)h * D + d] = den > 0.f ? num / den * v_scale : 0.f;
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

size_t gqa_fp8_smem_bytes() { return sizeof(Fp8Smem) + 1024; }

bool gqa_fp8_supported(const Problem &pr)
{
    // the in-kernel merge keeps G * splits weights in the stage ring
    return !pr.latent && pr.kv_planes == 2 && pr.dn == D && pr.HPU == G && pr.mpps > 0 &&
           (size_t)G * kMaxSplits * sizeof(float) <= sizeof(Fp8Smem::tiles);
}

cudaError_t launch_gqa_fp8(const DecodeArgs &a, float k_scale, float v_scale, cudaStream_t st)
{
    CUtensorMap map;
    const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)a.NU, (cuuint64_t)a.num_pages * 2 * kPage};
    const cuuint64_t strides[2] = {(cuuint64_t)D, (cuuint64_t)a.NU * D};
    const cuuint32_t box[3] = {(cuuint32_t)D, 1, (cuuint32_t)kPage};
    if (encode_tiled(&map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<__nv_bfloat16 *>(a.kv), dims, strides, box,
                     CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    const size_t smem = gqa_fp8_smem_bytes();
    cudaError_t e =
        cudaFuncSetAttribute(gqa_fp8_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess)
        return e;
    gqa_fp8_decode_kernel<<<dim3(a.num_splits, a.NU, a.B), THREADS, smem, st>>>(map, a, a.scale_log2 * k_scale,
                                                                                v_scale);
    return cudaGetLastError();
}

}  // namespace kvattn
