// The steps either side of decode attention.
//
// Before attention: the rotary position embedding of the position branch
// (MLA explainer, mlqm.cn/news/371735, section 2.2: q^R and k^R are rotated,
// the semantic parts are not), the new token's [latent ; k^R] row appended to
// the paged cache (section 2.4: the compact latent is what is cached), and the
// query absorption of the key up-projection (MLRA page, aitntnews.com
// newId=23265, MLA paragraph: W_UK folds into the query at decode time).
// After attention: the up-projection by W_UV (section 2.3: the output weights
// the semantic values c W_UV), for MLRA with one W_UV block per branch so the
// branch sum is part of the contraction (MLRA page, "moving the sum
// outside").
//
// RoPE (the pages print no formula): consecutive pairs (x[2i], x[2i+1]) of a
// d-wide slice turned by pos * base^(-2i/d), the rotary embedding's original
// form.  The angle and the turn are computed in double precision and rounded
// once to bf16 (round to nearest even).
//
// The projections are per-head GEMMs y[r][h] = x[r][h] W[h] on the tensor
// cores: one CTA per (head, 64..256 output columns, 128 rows), x and W tiles
// staged by TMA in 64-wide chunks of the contraction, tcgen05 MMAs
// (M = 128, K = 16) accumulating in TMEM, fp32 read back for the epilogue.
// Both are bound by reading W (tens of MB) from HBM.
#include <math.h>

#include "kvattn_internal.cuh"
#include "sm100.cuh"

namespace kvattn {

namespace {

bool is_aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// ------------------------------------------------------------------- RoPE

// Turn the pair (x0, x1), pair index i of a d-wide slice, at position pos.
__device__ __forceinline__ __nv_bfloat162 rope_pair(__nv_bfloat162 v, long long pos, int i, int d, double log2_base)
{
    const double inv_freq = exp2(-2.0 * (double)i / (double)d * log2_base);
    double s, c;
    sincos((double)pos * inv_freq, &s, &c);
    const double x0 = (double)__bfloat162float(v.x), x1 = (double)__bfloat162float(v.y);
    __nv_bfloat162 r;
    r.x = __double2bfloat16(x0 * c - x1 * s);
    r.y = __double2bfloat16(x0 * s + x1 * c);
    return r;
}

// One thread per pair: row = t / (rd / 2), pair = t % (rd / 2).
__global__ void rope_kernel(__nv_bfloat16 *x, long long rows, int row_elems, int off, int rd, int rows_per_pos,
                            const int32_t *pos, double log2_base)
{
    const int half = rd / 2;
    for (long long t = blockIdx.x * (long long)blockDim.x + threadIdx.x; t < rows * half;
         t += (long long)gridDim.x * blockDim.x) {
        const long long row = t / half;
        const int i = (int)(t % half);
        __nv_bfloat162 *p = reinterpret_cast<__nv_bfloat162 *>(x + row * row_elems + off) + i;
        *p = rope_pair(*p, pos[row / rows_per_pos], i, rd, log2_base);
    }
}

// ------------------------------------------------------------ cache append

struct AppendArgs {
    const __nv_bfloat16 *src;     // [B*Q][row] latent, or [B*Q][2][row] K, V (GQA/MQA)
    const int32_t *pos;           // [B*Q]
    const int32_t *block_table;   // nullptr: contiguous
    __nv_bfloat16 *cache;
    int32_t *err;                 // may be null
    int q_len, mpps, num_pages;
    int row;                      // elements per token row (per plane for GQA/MQA)
    int copy;                     // leading elements copied as they are (latent part)
    int rot_width, rot_count;     // RoPE over rot_count slices of rot_width after `copy` (0: none)
    int planes;                   // 1 (latent) or 2 (K and V planes of GQA/MQA)
    double log2_base;
};

// One CTA per new token: resolve its page and slot, copy the row with 16-byte
// vectors, turn the rope slices pair by pair.
__global__ void append_kernel(const AppendArgs a)
{
    const int t = blockIdx.x;
    const int s = t / a.q_len;
    const long long p = a.pos[t];
    if (p < 0 || p >= (long long)a.mpps * kPage) {
        if (threadIdx.x == 0 && a.err)
            atomicOr(a.err, KVATTN_DEVERR_POS_OUT_OF_RANGE);
        return;
    }
    const long long pi = p / kPage;
    const long long page = a.block_table ? (long long)a.block_table[(long long)s * a.mpps + pi]
                                         : (long long)s * a.mpps + pi;
    if (page < 0 || page >= a.num_pages) {
        if (threadIdx.x == 0 && a.err)
            atomicOr(a.err, KVATTN_DEVERR_PAGE_OUT_OF_RANGE);
        return;
    }
    const int slot = (int)(p % kPage);
    for (int pl = 0; pl < a.planes; ++pl) {
        const __nv_bfloat16 *src = a.src + ((long long)t * a.planes + pl) * a.row;
        __nv_bfloat16 *dst = a.cache + ((page * a.planes + pl) * kPage + slot) * (long long)a.row;
        // K of GQA/MQA (plane 0) is turned whole; V (plane 1) and the latent are copied
        const bool turn = a.rot_count > 0 && (a.planes == 1 || pl == 0);
        const int copy = a.planes == 1 ? a.copy : (turn ? 0 : a.row);
        for (int i = threadIdx.x; i < copy / 8; i += blockDim.x)
            reinterpret_cast<uint4 *>(dst)[i] = reinterpret_cast<const uint4 *>(src)[i];
        if (turn) {
            const int half = a.rot_width / 2;
            for (int i = threadIdx.x; i < a.rot_count * half; i += blockDim.x) {
                const int off = copy + (i / half) * a.rot_width;
                const __nv_bfloat162 v = reinterpret_cast<const __nv_bfloat162 *>(src + off)[i % half];
                reinterpret_cast<__nv_bfloat162 *>(dst + off)[i % half] = rope_pair(v, p, i % half, a.rot_width,
                                                                                    a.log2_base);
            }
        } else if (a.planes == 1) {
            for (int i = copy + threadIdx.x; i < a.row; i += blockDim.x)
                dst[i] = src[i];
        }
    }
}

// ------------------------------------------------------- head projection

constexpr int kHpThreads = 128;
constexpr int kHpStages = 4;
constexpr int kHpChunk = 64;                       // contraction elements per stage (128-byte rows)
constexpr int kHpXBytes = 128 * kHpChunk * 2;      // 128 rows x 64 (16 KB)
constexpr int kHpWBox = kHpChunk * 64 * 2;         // 64 contraction rows x 64 columns (8 KB)

// Shared memory of a head-projection CTA with `stages` ring slots (only as
// many as the contraction has chunks, so short contractions fit two CTAs on
// an SM): the x tiles, then the W tiles, then the barriers.
template <int NT>
struct HpLayout {
    static constexpr int kWStage = (NT / 64) * kHpWBox;
    __host__ __device__ static size_t w_off(int stages) { return (size_t)stages * kHpXBytes; }
    __host__ __device__ static size_t bar_off(int stages) { return w_off(stages) + (size_t)stages * kWStage; }
    __host__ __device__ static size_t bytes(int stages) { return bar_off(stages) + (2 * stages + 2) * 8; }
};

template <int NT>
constexpr uint32_t hp_tmem_cols()
{
    return NT <= 32 ? 32u : NT <= 64 ? 64u : NT <= 128 ? 128u : 256u;
}

// y[r][h][n0 .. n0+NT) = x[r][h][:] W[h][:][n0 .. n0+NT) for the 128 rows
// from m0.  Warp 0 streams x and W chunks, warp 1 issues the MMAs, then all
// four warps read the accumulator back (warp w owns TMEM lanes 32w..32w+31,
// i.e. rows m0 + 32w ..).  Rows past `rows` are zero-filled by TMA and not
// stored.
template <int NT>
__global__ void __launch_bounds__(kHpThreads)
    head_proj_kernel(const __grid_constant__ CUtensorMap xmap, const __grid_constant__ CUtensorMap wmap, void *y,
                     int out_fp32, int rows, int heads, int k, int n, int stages, int32_t *err)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    using Lay = HpLayout<NT>;
    unsigned char *xs = smem_raw;                                  // [stages][kHpXBytes]
    unsigned char *ws = smem_raw + Lay::w_off(stages);             // [stages][NT / 64][kHpWBox]
    uint64_t *full = reinterpret_cast<uint64_t *>(smem_raw + Lay::bar_off(stages));
    uint64_t *empty = full + stages;
    uint64_t *done = empty + stages;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(done + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = blockIdx.x, n0 = blockIdx.y * NT, m0 = blockIdx.z * 128;
    const int chunks = k / kHpChunk;
    constexpr uint32_t kCols = hp_tmem_cols<NT>();
    constexpr uint32_t kStageTx = kHpXBytes + Lay::kWStage;
    if (smem_u32(smem_raw) & 1023u) {
        if (threadIdx.x == 0 && err)
            atomicOr(err, KVATTN_DEVERR_WAIT_TIMEOUT);
        return;
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < stages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(done, 1);
        fence_mbar_init();
    }
    if (warp == 0)
        tmem_alloc(tmem_slot, kCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tacc = *tmem_slot;
    bool ok = true;

    if (warp == 0) {
        if (lane == 0) {
            prefetch_tmap(&xmap);
            prefetch_tmap(&wmap);
            int issued = 0;
            for (int c = 0; c < chunks; ++c) {
                const int st = c % stages;
                if (c >= stages && !mbar_wait(&empty[st], ((c / stages) - 1) & 1)) {
                    ok = false;
                    break;
                }
                mbar_arrive_expect_tx(&full[st], kStageTx);
                tma_load_3d(xs + (size_t)st * kHpXBytes, &xmap, c * kHpChunk, h, m0, &full[st]);
#pragma unroll
                for (int b = 0; b < NT / 64; ++b)
                    tma_load_2d(ws + (size_t)st * Lay::kWStage + b * kHpWBox, &wmap, n0 + 64 * b,
                                h * k + c * kHpChunk, &full[st]);
                issued = c + 1;
            }
            // every copy started here has landed before the CTA can exit
            for (int st = 0; st < stages && st < issued; ++st) {
                const int cl = st + ((issued - 1 - st) / stages) * stages;
                if (!mbar_wait(&full[st], (cl / stages) & 1))
                    ok = false;
            }
            if (!ok && err)
                atomicOr(err, KVATTN_DEVERR_WAIT_TIMEOUT);
        }
        __syncwarp();
    } else if (warp == 1) {
        constexpr uint32_t idesc = idesc_bf16_f32(128, NT, false, true);
        const uint64_t xdesc0 = smem_desc(smem_u32(xs), 16, 1024, 2);          // K-major rows of x
        const uint64_t wdesc0 = smem_desc(smem_u32(ws), kHpWBox, 1024, 2);     // N-major rows of W
        for (int c = 0; c < chunks; ++c) {
            const int st = c % stages;
            if (!__all_sync(0xffffffffu, mbar_wait(&full[st], (c / stages) & 1))) {
                ok = false;
                break;
            }
            tc_fence_after();
            if (lane == 0) {
                const uint64_t xd = xdesc0 + (uint64_t)(st * (kHpXBytes >> 4));
                const uint64_t wd = wdesc0 + (uint64_t)(st * (Lay::kWStage >> 4));
#pragma unroll
                for (int k16 = 0; k16 < kHpChunk / 16; ++k16)
                    umma_ss(tacc, xd + (uint64_t)(k16 * 2), wd + (uint64_t)(k16 * 128), idesc, (c | k16) ? 1u : 0u);
                umma_commit(&empty[st]);
            }
            __syncwarp();
        }
        if (lane == 0)
            umma_commit(done);
        __syncwarp();
        if (!ok && lane == 0 && err)
            atomicOr(err, KVATTN_DEVERR_WAIT_TIMEOUT);
    }

    // epilogue: row m0 + threadIdx.x, NT columns from TMEM
    const bool have = __all_sync(0xffffffffu, mbar_wait(done, 0));
    tc_fence_after();
    const int row = m0 + threadIdx.x;
    const uint32_t lane_addr = (uint32_t)(warp * 32) << 16;
    const size_t base = ((size_t)row * heads + h) * n + n0;
#pragma unroll 1
    for (int c = 0; c < NT / 32; ++c) {
        uint32_t r[32];
        if (have)
            tmem_ld32(tacc + lane_addr + 32 * c, r);
        if (row < rows) {
            if (out_fp32) {
                float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(y) + base + 32 * c);
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    dst[i] = have ? make_float4(__uint_as_float(r[4 * i]), __uint_as_float(r[4 * i + 1]),
                                                __uint_as_float(r[4 * i + 2]), __uint_as_float(r[4 * i + 3]))
                                  : make_float4(0.f, 0.f, 0.f, 0.f);
            } else {
                uint4 *dst = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(y) + base + 32 * c);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    uint32_t pk[4];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const __nv_bfloat162 v = __floats2bfloat162_rn(have ? __uint_as_float(r[8 * i + 2 * j]) : 0.f,
                                                                       have ? __uint_as_float(r[8 * i + 2 * j + 1]) : 0.f);
                        pk[j] = *reinterpret_cast<const uint32_t *>(&v);
                    }
                    dst[i] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                }
            }
        }
    }
    if (!have && threadIdx.x == 0 && err)
        atomicOr(err, KVATTN_DEVERR_WAIT_TIMEOUT);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0)
        tmem_dealloc(tacc, kCols);
}

template <int NT>
cudaError_t launch_head_proj(const CUtensorMap &xm, const CUtensorMap &wm, void *y, int out_fp32, int rows, int heads,
                             int k, int n, int32_t *err, cudaStream_t st)
{
    const int chunks = k / kHpChunk;
    const int stages = chunks < kHpStages ? chunks : kHpStages;
    const size_t smem = HpLayout<NT>::bytes(stages);
    cudaError_t e =
        cudaFuncSetAttribute(head_proj_kernel<NT>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess)
        return e;
    const dim3 grid(heads, n / NT, (rows + 127) / 128);
    head_proj_kernel<NT><<<grid, kHpThreads, smem, st>>>(xm, wm, y, out_fp32, rows, heads, k, n, stages, err);
    return cudaGetLastError();
}

}  // namespace

}  // namespace kvattn

using namespace kvattn;

extern "C" int kvattn_rope(void *x, int32_t rows, int32_t row_elems, int32_t rot_offset, int32_t rot_dim,
                           int32_t rows_per_pos, const int32_t *pos, float rope_base, void *stream)
{
    if (!x || !pos || rows < 0 || row_elems < 2 || rot_dim < 2 || rot_dim % 2 || rot_offset < 0 ||
        rot_offset % 2 || row_elems % 2 || rot_offset + rot_dim > row_elems || rows_per_pos < 1 ||
        !(rope_base > 1.f) || !isfinite(rope_base))
        return KVATTN_ERR_INVALID_ARG;
    if (!is_aligned(x, 4) || !is_aligned(pos, 4))
        return KVATTN_ERR_MISALIGNED;
    if (rows == 0)
        return KVATTN_OK;
    const long long pairs = (long long)rows * (rot_dim / 2);
    const int threads = 256;
    const long long blocks = (pairs + threads - 1) / threads;
    const int grid = (int)(blocks < 148LL * 16 ? blocks : 148LL * 16);
    rope_kernel<<<grid, threads, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<__nv_bfloat16 *>(x), rows, row_elems, rot_offset, rot_dim, rows_per_pos, pos,
        log2((double)rope_base));
    return cudaGetLastError() == cudaSuccess ? KVATTN_OK : KVATTN_ERR_CUDA;
}

extern "C" int kvattn_append_kv(int32_t variant, const kvattn_params *p, const void *new_kv, const int32_t *pos,
                                const int32_t *block_table, void *kv_cache, float rope_base, int32_t *device_error,
                                void *stream)
{
    Problem pr;
    const int st = validate_params(variant, p, &pr);
    if (st)
        return st;
    if (!new_kv || !pos || !kv_cache)
        return KVATTN_ERR_INVALID_ARG;
    if (p->cache_dtype != KVATTN_CACHE_BF16)
        return KVATTN_ERR_UNSUPPORTED;      // rows are appended in bf16
    if (!(rope_base == 0.f || (rope_base > 1.f && isfinite(rope_base))))
        return KVATTN_ERR_INVALID_ARG;
    if (!is_aligned(new_kv, 16) || !is_aligned(kv_cache, 16) || !is_aligned(pos, 4) ||
        (block_table && !is_aligned(block_table, 4)) || (device_error && !is_aligned(device_error, 4)))
        return KVATTN_ERR_MISALIGNED;
    AppendArgs a{};
    a.src = static_cast<const __nv_bfloat16 *>(new_kv);
    a.pos = pos;
    a.block_table = block_table;
    a.cache = static_cast<__nv_bfloat16 *>(kv_cache);
    a.err = device_error;
    a.q_len = pr.q_len;
    a.mpps = pr.mpps;
    a.num_pages = pr.num_pages;
    a.row = pr.row;
    a.log2_base = rope_base > 0.f ? log2((double)rope_base) : 0.0;
    if (pr.latent) {
        a.planes = 1;
        a.copy = pr.NU * pr.dn;
        a.rot_width = pr.dr;
        a.rot_count = (rope_base > 0.f && pr.dr > 0) ? 1 : 0;
    } else if (pr.kv_planes == 1) {
        // tied keys and values (GTA, MFA-KR): the row is the value too, so it
        // is stored as given (the pages do not place RoPE for the tie)
        if (rope_base != 0.f)
            return KVATTN_ERR_INVALID_ARG;
        a.planes = 1;
        a.copy = pr.row;
        a.rot_width = 0;
        a.rot_count = 0;
    } else {
        a.planes = 2;
        a.copy = 0;
        a.rot_width = pr.dn;
        a.rot_count = rope_base > 0.f ? pr.NU : 0;
    }
    append_kernel<<<pr.B, 128, 0, static_cast<cudaStream_t>(stream)>>>(a);
    return cudaGetLastError() == cudaSuccess ? KVATTN_OK : KVATTN_ERR_CUDA;
}

extern "C" int kvattn_head_proj(const void *x, const void *w, void *y, int32_t out_dtype, int32_t rows,
                                int32_t heads, int32_t k, int32_t n, int32_t *device_error, void *stream)
{
    if (!x || !w || !y || rows < 0 || heads < 1 || k < 64 || k % 64 || n < 64 || n % 64)
        return KVATTN_ERR_INVALID_ARG;
    if (out_dtype != KVATTN_OUT_BF16 && out_dtype != KVATTN_OUT_FP32)
        return KVATTN_ERR_INVALID_ARG;
    if ((long long)heads * k > (1LL << 31) || (long long)rows * heads > (1LL << 31) || n > (1 << 20) ||
        rows > 65535 * 128)
        return KVATTN_ERR_UNSUPPORTED;
    if (!is_aligned(x, 16) || !is_aligned(w, 16) || !is_aligned(y, 16) ||
        (device_error && !is_aligned(device_error, 4)))
        return KVATTN_ERR_MISALIGNED;
    if (rows == 0)
        return KVATTN_OK;
    CUtensorMap xm, wm;
    {
        const cuuint64_t dims[3] = {(cuuint64_t)k, (cuuint64_t)heads, (cuuint64_t)rows};
        const cuuint64_t strides[2] = {(cuuint64_t)k * 2, (cuuint64_t)heads * k * 2};
        const cuuint32_t box[3] = {kHpChunk, 1, 128};
        if (encode_tiled(&xm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(x), dims, strides, box,
                         CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
            return KVATTN_ERR_UNSUPPORTED;
    }
    {
        const cuuint64_t dims[2] = {(cuuint64_t)n, (cuuint64_t)heads * k};
        const cuuint64_t strides[1] = {(cuuint64_t)n * 2};
        const cuuint32_t box[2] = {64, kHpChunk};
        if (encode_tiled(&wm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(w), dims, strides, box,
                         CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
            return KVATTN_ERR_UNSUPPORTED;
    }
    const int fp32 = out_dtype == KVATTN_OUT_FP32;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // the widest output tile that still gives about 1.5 CTAs per SM (the
    // work is a stream of W; narrow tiles re-read x, wide tiles leave SMs idle)
    const long long per_tile = (long long)heads * ((rows + 127) / 128);
    const long long want = 3LL * sm_count() / 2;
    int nt = 64;
    if (n % 256 == 0 && per_tile * (n / 256) >= want)
        nt = 256;
    else if (n % 128 == 0 && per_tile * (n / 128) >= want)
        nt = 128;
    cudaError_t e;
    if (nt == 256)
        e = launch_head_proj<256>(xm, wm, y, fp32, rows, heads, k, n, device_error, s);
    else if (nt == 128)
        e = launch_head_proj<128>(xm, wm, y, fp32, rows, heads, k, n, device_error, s);
    else
        e = launch_head_proj<64>(xm, wm, y, fp32, rows, heads, k, n, device_error, s);
    return e == cudaSuccess ? KVATTN_OK : KVATTN_ERR_CUDA;
}
