// Absorbed MLA decode on a pair of CTAs (a 2-CTA cluster) on the tensor cores.
//
// MLA decodes as one 576-wide MQA head whose value is the 512-wide latent
// (MLRA page: the MLA paragraph on absorbing W_UK into the query; MLA
// explainer section 2.3 formula, section 2.2 concatenation).  A 128-head x
// 512 fp32 output would fill all of one SM's TMEM, so the two CTAs of a
// cluster each own half of the value columns.  Instead of both forming the
// full 128 x T score tile, they split its 576-wide contraction:
//
//   rank 0: key columns   0..255  (latent)          value columns   0..255
//   rank 1: key columns 256..575  (latent + rope)   value columns 256..511
//
// Each rank loads only its own key columns of every tile (4 or 5 boxes of
// 64), computes a partial score S_r = Q[:, cols_r] K[:, cols_r]^T with a
// tcgen05 MMA into TMEM, and sends its partial to the other rank's shared
// memory (distributed shared memory, remote mbarrier arrive).  Both ranks
// then hold S = S_0 + S_1 bit for bit (fp32 addition is commutative), run the
// same online softmax and accumulate P V over their own value columns.  The
// tensor work and the cache bytes per rank are halves of the whole, with no
// score computed twice.
//
// Roles per CTA (320 threads): warp 0 TMEM allocation and TMA producer,
// warp 1 MMA issue, warps 2-9 softmax (two threads per head row, each owning
// half of the tile's columns and half of the output columns).  Every wait is
// bounded; the CTAs meet at a cluster barrier before exit so that no remote
// access can reach a finished CTA.
#include <math.h>

#include "latent_common.cuh"

namespace kvattn {

namespace {

using namespace latent;

constexpr int T = 64;                      // tokens per tile (one page)
constexpr int STAGES = 3;
constexpr int NKB_MAX = 5;                 // rank 1: 4 latent boxes + the rope box
constexpr int NVB = 4;                     // 256 value columns per rank
constexpr int NQT = 4;                     // latent query chunks held in TMEM
constexpr int kSoftmaxThreads = 256;
constexpr int kThreads = 64 + kSoftmaxThreads;
constexpr int kBoxBytes = T * 128;
constexpr int kStageBytes = NKB_MAX * kBoxBytes;
constexpr int kDvSlot = NVB * 64;
constexpr int TH = T / 2;                  // score columns per softmax thread
constexpr int OH = kDvSlot / 2;            // output columns per softmax thread

struct PairSmem {
    unsigned char qr[kQChunkBytes];          // rope query chunk (rank 1), K-major, 128-byte swizzle
    unsigned char kv[STAGES][kStageBytes];
    float recv[2][kRows][T];                 // the other rank's partial scores [parity][row][token]
    float xmax[2][2][kRows];                 // [exchange parity][column half][row]
    uint32_t pvalid[kMaxSplitPages / 32];
    uint64_t kv_full[STAGES];
    uint64_t kv_empty[STAGES];
    uint64_t s_full[2];
    uint64_t p_full[2];
    uint64_t xfull[2];                       // the other rank's partial scores have arrived
    uint64_t o_ready;
    uint64_t q_ready;
    uint64_t mma_done;
    uint64_t xbar[4];
    uint32_t tmem_base;
};

__global__ void __launch_bounds__(kThreads, 1) mla_pair_kernel(const __grid_constant__ CUtensorMap kv_map,
                                                               const DecodeArgs a)
{
    constexpr uint32_t kTmemCols = 512;
    constexpr uint32_t kIdescS = idesc_bf16_f32(kRows, T, false, false);
    constexpr uint32_t kIdescPV = idesc_bf16_f32(kRows, kDvSlot, false, true);
    static_assert(2 * T + kDvSlot + NQT * 32 <= 512, "TMEM budget");

    extern __shared__ __align__(1024) unsigned char smem_raw[];
    PairSmem &S = *reinterpret_cast<PairSmem *>(smem_raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int split = blockIdx.x, b = blockIdx.z;
    const uint32_t rank = cluster_ctarank();          // value half
    const uint32_t peer = rank ^ 1u;
    const int nkb = 4 + (int)rank;
    if (smem_u32(smem_raw) & 1023u) {
        // both CTAs share the launch's shared-memory layout, so both stop here
        if (threadIdx.x == 0)
            raise_error(a.err, KVATTN_DEVERR_WAIT_TIMEOUT);
        return;
    }

    int L = a.seq_lens[b];
    if (L > a.max_seq_len) {
        if (threadIdx.x == 0 && split == 0 && rank == 0)
            raise_error(a.err, KVATTN_DEVERR_SEQ_TOO_LONG);
        L = a.max_seq_len;
    }
    L = max(L, 0);
    const int p0 = split * a.pages_per_split;
    const int tok_end = min(L, (p0 + a.pages_per_split) * kPage);
    const int n = tok_end > p0 * kPage ? (tok_end - p0 * kPage + T - 1) / T : 0;

    if (threadIdx.x == 0) {
        for (int st = 0; st < STAGES; ++st) {
            mbar_init(&S.kv_full[st], 1);
            mbar_init(&S.kv_empty[st], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&S.s_full[i], 1);
            mbar_init(&S.p_full[i], kSoftmaxThreads);
            mbar_init(&S.xfull[i], kSoftmaxThreads / 32);
        }
        mbar_init(&S.o_ready, 1);
        mbar_init(&S.q_ready, kSoftmaxThreads);
        mbar_init(&S.mma_done, 1);
        for (int q = 0; q < 4; ++q)
            mbar_init(&S.xbar[q], 64);
        fence_mbar_init();
    }
    if (warp == 0)
        tmem_alloc(&S.tmem_base, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    cluster_sync_all();      // the other rank's barriers exist before anything is sent to them
    const uint32_t tbase = S.tmem_base;
    const uint32_t tS = tbase;             // 2 score / probability buffers of T columns
    const uint32_t tO = tbase + 2 * T;     // 256 output columns
    const uint32_t tQ = tO + kDvSlot;      // 4 latent query chunks (bf16 pairs)

    if (warp == 0) {
        // ---------------------------------------------------------------- TMA
        if (lane == 0 && n > 0) {
            prefetch_tmap(&kv_map);
            int issued = 0;
            for (int j = 0; j < n; ++j) {
                const int st = j % STAGES;
                if (j >= STAGES && !mbar_wait(&S.kv_empty[st], ((j / STAGES) - 1) & 1)) {
                    raise_error(a.err, KVATTN_DEVERR_WAIT_TIMEOUT);
                    break;
                }
                issued = j + 1;
                const int tok0 = p0 * kPage + j * T;
                const long long page = page_id(a, b, tok0 / kPage);
                if (!page_ok(a, page)) {
                    if (rank == 0)
                        raise_error(a.err, KVATTN_DEVERR_PAGE_OUT_OF_RANGE);
                    mbar_arrive(&S.kv_full[st]);
                    continue;
                }
                mbar_arrive_expect_tx(&S.kv_full[st], (uint32_t)(nkb * kBoxBytes));
                const int y = (int)(page * kPage);
                for (int i = 0; i < nkb; ++i)
                    tma_load_2d(S.kv[st] + i * kBoxBytes, &kv_map, (int)rank * 256 + 64 * i, y, &S.kv_full[st]);
            }
            for (int st = 0; st < STAGES && st < issued; ++st) {
                const int jl = st + ((issued - 1 - st) / STAGES) * STAGES;
                if (!mbar_wait(&S.kv_full[st], (jl / STAGES) & 1))
                    raise_error(a.err, KVATTN_DEVERR_WAIT_TIMEOUT);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA
        const uint32_t qrbase = smem_u32(S.qr);
        bool ok = mbar_wait(&S.q_ready, 0);
        tc_fence_after();
        auto issue_pv = [&](int t) -> bool {
            if (!mbar_wait(&S.p_full[t & 1], (t >> 1) & 1))
                return false;
            tc_fence_after();
            if (lane == 0) {
                const uint32_t vbase = smem_u32(S.kv[t % STAGES]);
#pragma unroll
                for (int k = 0; k < T / 16; ++k) {
                    const uint64_t vd = smem_desc(vbase + k * 16 * 128, kBoxBytes, 1024, 2);
                    umma_ts(tO, tS + (t & 1) * T + 8 * k, vd, kIdescPV, (t > 0 || k > 0) ? 1u : 0u);
                }
                umma_commit(&S.o_ready);
                umma_commit(&S.kv_empty[t % STAGES]);
            }
            __syncwarp();
            return true;
        };
        int j = 0;
        for (; ok && j < n; ++j) {
            const int st = j % STAGES;
            if (!mbar_wait(&S.kv_full[st], (j / STAGES) & 1)) {
                ok = false;
                break;
            }
            const int ntok = tile_ntok<T>(S.pvalid, L, p0, j);
            if (ntok < T) {
                const int rows = T - ntok;
                for (int idx = lane; idx < rows * nkb * 8; idx += 32) {
                    const int box = idx / (rows * 8), rem = idx % (rows * 8);
                    const int row = ntok + rem / 8, piece = rem % 8;
                    *reinterpret_cast<uint4 *>(S.kv[st] + box * kBoxBytes + row * 128 + piece * 16) =
                        make_uint4(0, 0, 0, 0);
                }
                fence_proxy_async_smem();
                __syncwarp();
            }
            tc_fence_after();
            if (lane == 0) {
                const uint32_t kbase = smem_u32(S.kv[st]);
                for (int kb = 0; kb < nkb; ++kb) {
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const uint64_t kd = smem_desc(kbase + kb * kBoxBytes + k * 32, 16, 1024, 2);
                        if (kb < NQT) {
                            umma_ts(tS + (j & 1) * T, tQ + kb * 32 + k * 8, kd, kIdescS, (kb | k) ? 1u : 0u);
                        } else {
                            const uint64_t qd = smem_desc(qrbase + k * 32, 16, 1024, 2);
                            umma_ss(tS + (j & 1) * T, qd, kd, kIdescS, 1u);
                        }
                    }
                }
                umma_commit(&S.s_full[j & 1]);
            }
            __syncwarp();
            if (j >= 1 && !issue_pv(j - 1)) {
                ok = false;
                break;
            }
        }
        if (ok && n > 0 && !issue_pv(n - 1))
            ok = false;
        if (!ok && lane == 0)
            raise_error(a.err, KVATTN_DEVERR_WAIT_TIMEOUT);
        if (lane == 0)
            umma_commit(&S.mma_done);
        __syncwarp();
        if (!mbar_wait(&S.mma_done, 0) && lane == 0)
            raise_error(a.err, KVATTN_DEVERR_WAIT_TIMEOUT);
        __syncwarp();
    } else {
        // ------------------------------------------------------------ softmax
        const int sw = warp - 2;
        const int quarter = warp & 3;
        const int half = sw >> 2;
        const int h = quarter * 32 + lane;
        const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
        const bool valid = h < a.H;
        {
            const int npg = min(a.pages_per_split, max(0, (L + kPage - 1) / kPage - p0));
            fill_page_bits(S.pvalid, a, b, p0, npg, threadIdx.x - 64, kSoftmaxThreads);
            // this rank's query columns: latent [256 rank, 256 rank + 256) to TMEM,
            // and for rank 1 the rope query to shared memory
            const __nv_bfloat16 *qn = valid ? a.q_nope + ((size_t)b * a.H + h) * a.dn + rank * 256 : nullptr;
            const __nv_bfloat16 *qr = valid ? a.q_rope + ((size_t)b * a.H + h) * a.dr : nullptr;
#pragma unroll 1
            for (int kb = half; kb < NQT; kb += 2) {
                uint32_t r[32];
#pragma unroll
                for (int p = 0; p < 8; ++p) {
                    const uint4 v = qn ? *reinterpret_cast<const uint4 *>(qn + 64 * kb + 8 * p) : make_uint4(0, 0, 0, 0);
                    r[4 * p] = v.x;
                    r[4 * p + 1] = v.y;
                    r[4 * p + 2] = v.z;
                    r[4 * p + 3] = v.w;
                }
                tmem_st32(tQ + lane_addr + kb * 32, r);
            }
            if (rank == 1 && half == 0) {
#pragma unroll
                for (int p = 0; p < 8; ++p) {
                    const uint4 v = qr ? *reinterpret_cast<const uint4 *>(qr + 8 * p) : make_uint4(0, 0, 0, 0);
                    *reinterpret_cast<uint4 *>(&S.qr[h * 128 + ((p ^ (h & 7)) << 4)]) = v;
                }
            }
            fence_proxy_async_smem();
            named_sync(1, kSoftmaxThreads);
            tc_fence_before();
            mbar_arrive(&S.q_ready);
        }

        const uint32_t peer_xfull0 = mapa_shared(smem_u32(&S.xfull[0]), peer);
        const uint32_t peer_xfull1 = mapa_shared(smem_u32(&S.xfull[1]), peer);
        float m_ref = -INFINITY, l = 0.f;
        bool ok = true;
        for (int j = 0; j < n; ++j) {
            const int sb = j & 1;
            ok = __all_sync(0xffffffffu, mbar_wait(&S.s_full[sb], (j >> 1) & 1));
            if (!ok)
                break;
            tc_fence_after();
            float s[TH];
            {
                uint32_t r[TH];
                tmem_ld32(tS + lane_addr + sb * T + half * TH, r);
#pragma unroll
                for (int i = 0; i < TH; ++i)
                    s[i] = __uint_as_float(r[i]);
            }
            // send this rank's partial scores to the other rank, take its partial
            {
                const uint32_t dst = mapa_shared(smem_u32(&S.recv[sb][h][half * TH]), peer);
#pragma unroll
                for (int i = 0; i < TH; i += 4)
                    st_cluster_f32x4(dst + 4 * i, s[i], s[i + 1], s[i + 2], s[i + 3]);
                // one cluster-scope release per warp covers its lanes' stores (ordered
                // by the warp barrier), and one lane polls the local barrier
                __syncwarp();
                if (lane == 0)
                    mbar_arrive_cluster(sb ? peer_xfull1 : peer_xfull0);
                bool got = true;
                if (lane == 0)
                    got = mbar_wait_cluster(&S.xfull[sb], (j >> 1) & 1);
                ok = __shfl_sync(0xffffffffu, got ? 1 : 0, 0) != 0;
                __syncwarp();
                if (!ok)
                    break;
                const float4 *src = reinterpret_cast<const float4 *>(&S.recv[sb][h][half * TH]);
#pragma unroll
                for (int i = 0; i < TH / 4; ++i) {
                    const float4 v = src[i];
                    s[4 * i] += v.x;
                    s[4 * i + 1] += v.y;
                    s[4 * i + 2] += v.z;
                    s[4 * i + 3] += v.w;
                }
            }
#pragma unroll
            for (int i = 0; i < TH; ++i)
                s[i] *= a.scale_log2;
            const int ntok = tile_ntok<T>(S.pvalid, L, p0, j);
            if (ntok < T) {
#pragma unroll
                for (int i = 0; i < TH; ++i)
                    s[i] = half * TH + i < ntok ? s[i] : -INFINITY;
            }
            float mx8[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                mx8[q] = s[q];
#pragma unroll
                for (int i = q + 8; i < TH; i += 8)
                    mx8[q] = fmaxf(mx8[q], s[i]);
            }
            float mt = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                             fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
            S.xmax[sb][half][h] = mt;
            mbar_arrive(&S.xbar[quarter]);
            ok = __all_sync(0xffffffffu, mbar_wait(&S.xbar[quarter], j & 1));
            if (!ok)
                break;
            mt = fmaxf(mt, S.xmax[sb][half ^ 1][h]);

            float alpha = 1.f;
            bool rescale = false;
            if (mt > m_ref + kRescaleThreshold) {
                if (m_ref != -INFINITY) {
                    alpha = exp2f(m_ref - mt);
                    rescale = true;
                }
                m_ref = mt;
            }
            const float m_use = m_ref == -INFINITY ? 0.f : m_ref;
            float ps8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            uint32_t pk[TH / 2];
#pragma unroll
            for (int i = 0; i < TH / 2; ++i) {
                const float e0 = exp2f(s[2 * i] - m_use), e1 = exp2f(s[2 * i + 1] - m_use);
                ps8[i & 7] += e0 + e1;
                const __nv_bfloat162 v2 = __floats2bfloat162_rn(e0, e1);
                pk[i] = *reinterpret_cast<const uint32_t *>(&v2);
            }
            const float ps = ((ps8[0] + ps8[1]) + (ps8[2] + ps8[3])) + ((ps8[4] + ps8[5]) + (ps8[6] + ps8[7]));
            l = l * alpha + ps;
            tmem_st16(tS + lane_addr + sb * T + half * (TH / 2), pk);
            if (__any_sync(0xffffffffu, rescale)) {
                ok = __all_sync(0xffffffffu, mbar_wait(&S.o_ready, (j - 1) & 1));
                if (!ok)
                    break;
                tc_fence_after();
                uint32_t r[32];
#pragma unroll 1
                for (int c = 0; c < OH / 32; ++c) {
                    const uint32_t o_addr = tO + lane_addr + half * OH + 32 * c;
                    tmem_ld32(o_addr, r);
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
                    tmem_st32(o_addr, r);
                }
            }
            tc_fence_before();
            mbar_arrive(&S.p_full[sb]);
        }
        if (!ok && lane == 0)
            raise_error(a.err, KVATTN_DEVERR_WAIT_TIMEOUT);

        if (ok) {
            S.xmax[n & 1][half][h] = l;
            mbar_arrive(&S.xbar[quarter]);
            ok = __all_sync(0xffffffffu, mbar_wait(&S.xbar[quarter], n & 1));
            if (ok)
                l += S.xmax[n & 1][half ^ 1][h];
            else if (lane == 0)
                raise_error(a.err, KVATTN_DEVERR_WAIT_TIMEOUT);
        }
        bool have = false;
        if (ok && n > 0) {
            have = __all_sync(0xffffffffu, mbar_wait(&S.o_ready, (n - 1) & 1));
            if (!have && lane == 0)
                raise_error(a.err, KVATTN_DEVERR_WAIT_TIMEOUT);
            tc_fence_after();
        }
        const size_t prow = ((size_t)b * a.num_splits + split) * a.HU + (valid ? h : 0);
        float *dst = a.po + prow * a.dn + rank * kDvSlot + half * OH;
        const float inv = (have && l > 0.f) ? 1.f / l : 0.f;
        uint32_t r[64];
#pragma unroll 1
        for (int c = 0; c < OH / 64; ++c) {
            if (have)
                tmem_ld64(tO + lane_addr + half * OH + 64 * c, r);
            if (valid) {
#pragma unroll
                for (int i = 0; i < 64; i += 4) {
                    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
                    if (have)
                        v = make_float4(__uint_as_float(r[i]) * inv, __uint_as_float(r[i + 1]) * inv,
                                        __uint_as_float(r[i + 2]) * inv, __uint_as_float(r[i + 3]) * inv);
                    *reinterpret_cast<float4 *>(dst + 64 * c + i) = v;
                }
            }
        }
        if (valid && half == 0 && rank == 0)
            a.plse[prow] = (have && l > 0.f) ? (m_ref + log2f(l)) * kLn2 : -INFINITY;
    }
    __syncwarp();

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0)
        tmem_dealloc(tbase, kTmemCols);
    cluster_sync_all();      // no remote store or arrive can reach a CTA that has exited
}

}  // namespace

// MLA with a 512-wide latent and a 64-wide rope key, at most 128 heads.
bool mla_pair_supported(const Problem &pr)
{
    return pr.latent && !pr.mlra && pr.NU == 1 && pr.dn == 512 && pr.dr == 64 && pr.H <= kRows;
}

cudaError_t launch_mla_pair(const DecodeArgs &a, cudaStream_t st)
{
    CUtensorMap map;
    const cuuint64_t dims[2] = {(cuuint64_t)a.row, (cuuint64_t)a.num_pages * kPage};
    const cuuint64_t strides[1] = {(cuuint64_t)a.row * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)T};
    if (encode_tiled(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<__nv_bfloat16 *>(a.kv), dims, strides,
                     box, CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    const size_t smem = sizeof(PairSmem);
    cudaError_t e = cudaFuncSetAttribute(mla_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess)
        return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(a.num_splits, 2, a.B);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = 2;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, mla_pair_kernel, map, a);
    if (e != cudaSuccess)
        return e;
    return cudaGetLastError();
}

}  // namespace kvattn
