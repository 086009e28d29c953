// Latent decode on the 5th-generation tensor cores: GLA and MLRA (and their
// single-group or single-branch shards).
//
// Every query head scores the same cached latent rows (GLA page: one latent
// head per query group; MLRA page: the latent split into branches attended on
// their own, branch outputs summed afterwards), so the scores and P.V are real
// [heads x K] x [K x tokens] contractions and run as tcgen05 MMAs with fp32
// accumulators in TMEM.  (Absorbed MLA, one 512-wide latent, runs on the
// 2-CTA kernel in decode_mla_pair.cu.)
//
// One CTA owns (part s of the context, slot, sequence b).  A slot is a latent
// group for GLA (its heads padded to the MMA's 128 rows) and a branch for
// MLRA (all heads, each with its own query slice).  Key columns of the slot
// are [latent slice | shared rope key], each a 64-column box of the page row.
//
// The query rows are the MMA's A operand for every tile.  Their first NQT
// 64-column chunks sit in TMEM (an A operand in TMEM costs no shared-memory
// bandwidth), the rest in shared memory.  TMEM columns: two score /
// probability buffers of T, the output slice, the Q chunks.
//
// Warp roles (320 threads):
//   warp 0     TMEM allocation; one thread streams the tiles into a
//              STAGES-deep ring with 2-D TMA loads (128-byte swizzle; a
//              128-token tile is two pages)
//   warp 1     one thread issues S_j = Q K_j^T into one of two TMEM score
//              buffers, then P_{j-1} V_{j-1} into the TMEM output; the warp
//              zeroes the rows of a tile past the context first (0 * NaN
//              would poison the MMA)
//   warps 2-9  two threads per head row, each owning half of the tile's
//              columns and half of O's: read S_j from TMEM, exchange the tile
//              maximum with the partner thread through shared memory, online
//              softmax in fp32 (base 2) with a lazy rescale (the reference
//              max moves only when a score exceeds it by more than 2^8, so O
//              is rarely touched), write P_j as bf16 into the score buffer it
//              came from (the A operand of the P.V MMA), and at the end
//              normalise O and write the part result and its lse.
// Every wait is bounded; a wait that gives up sets an error bit and the CTA
// drains its own copies and MMAs before it frees TMEM and exits.
#include <math.h>

#include <type_traits>

#include "latent_common.cuh"

namespace kvattn {

namespace {

using namespace latent;

constexpr int kSoftmaxThreads = 256;       // two warps per TMEM lane quarter
constexpr int kThreads = 64 + kSoftmaxThreads;

template <int T, int NKB, int STAGES, int NQT>
struct LatentSmem {
    static constexpr int kBoxBytes = T * 128;
    static constexpr int kStageBytes = NKB * kBoxBytes;
    static constexpr int kQSmem = NKB - NQT > 0 ? NKB - NQT : 1;
    unsigned char q[kQSmem][kQChunkBytes];    // Q chunks NQT..NKB-1 (K-major, 128-byte swizzle)
    unsigned char kv[STAGES][kStageBytes];
    float xmax[2][2][kRows];                  // [exchange parity][column half][row]
    uint32_t pvalid[kMaxSplitPages / 32];     // one bit per page of the part
    uint64_t full[STAGES];                    // the stage's boxes landed
    uint64_t empty[STAGES];                   // P.V done with the stage
    uint64_t s_full[2];
    uint64_t p_full[2];
    uint64_t o_ready;
    uint64_t q_ready;
    uint64_t mma_done;
    uint64_t xbar[4];                         // per lane quarter: the two threads of a row meet here
    uint32_t tmem_base;
};

template <int T, int NKB, int NVB, int STAGES, int NQT>
__global__ void __launch_bounds__(kThreads, 1)
    latent_tc_decode_kernel(const __grid_constant__ CUtensorMap kv_map, const DecodeArgs a)
{
    using Smem = LatentSmem<T, NKB, STAGES, NQT>;
    constexpr int kBoxBytes = Smem::kBoxBytes;
    constexpr int kDvSlot = NVB * 64;                            // value columns of this CTA
    constexpr int kColsUsed = 2 * T + kDvSlot + NQT * 32;
    static_assert(kColsUsed <= 512, "TMEM budget");
    constexpr uint32_t kTmemCols = kColsUsed <= 256 ? 256 : 512;
    constexpr uint32_t kIdescS = idesc_bf16_f32(kRows, T, false, false);
    constexpr uint32_t kIdescPV = idesc_bf16_f32(kRows, kDvSlot, false, true);

    extern __shared__ __align__(1024) unsigned char smem_raw[];
    Smem &S = *reinterpret_cast<Smem *>(smem_raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int split = blockIdx.x, slot = blockIdx.y, b = blockIdx.z;
    pdl_launch_dependents();
    if (smem_u32(smem_raw) & 1023u) {
        // the 128-byte swizzle atoms need 1024-byte alignment; never expected
        if (threadIdx.x == 0)
            raise_error(a.err, KVATTN_DEVERR_WAIT_TIMEOUT);
        return;
    }
    constexpr int NE = NKB - NVB;                                // rope boxes: stage positions 0..NE-1
    static_assert(NE == 1, "one 64-wide rope key box");
    // Key box (64-column block of the slot's key row) at stage position p:
    // the rope key first, then the slot's latent (value) columns.
    auto key_box = [&](int p) -> int { return p < NE ? NVB + p : p - NE; };

    const int L = row_context(a, b, threadIdx.x == 0 && split == 0 && slot == 0);
    const int p0 = split * a.pages_per_split;
    const int tok_end = min(L, (p0 + a.pages_per_split) * kPage);
    const int n = tok_end > p0 * kPage ? (tok_end - p0 * kPage + T - 1) / T : 0;

    if (threadIdx.x == 0) {
        for (int st = 0; st < STAGES; ++st) {
            mbar_init(&S.full[st], 1);
            mbar_init(&S.empty[st], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&S.s_full[i], 1);
            mbar_init(&S.p_full[i], kSoftmaxThreads);
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
    const uint32_t tbase = S.tmem_base;
    const uint32_t tS = tbase;                 // 2 score / probability buffers of T columns
    const uint32_t tO = tbase + 2 * T;         // kDvSlot output columns
    const uint32_t tQ = tO + kDvSlot;          // NQT query chunks of 32 columns (bf16 pairs)

    if (warp == 0) {
        // ---------------------------------------------------------------- TMA
        if (lane == 0 && n > 0) {
            prefetch_tmap(&kv_map);
            const int unit_col0 = slot * a.dn;
            constexpr int kSubs = T >= kPage ? T / kPage : 1;   // pages a tile spans
            constexpr int kSubRows = T >= kPage ? kPage : T;    // rows per TMA box
            int issued = 0;                                     // tiles whose loads were started
            for (; issued < n; ++issued) {
                const int j = issued, st = j % STAGES;
                if (j >= STAGES && !mbar_wait(&S.empty[st], ((j / STAGES) - 1) & 1)) {
                    raise_error(a.err, KVATTN_DEVERR_WAIT_TIMEOUT);
                    break;
                }
                // a tile with a bad page id loads nothing and only arrives
                const int tok0 = p0 * kPage + j * T;
                const int ntok = min(T, L - tok0);
                const int nsub = (ntok + kSubRows - 1) / kSubRows;  // boxes of this tile holding context
                long long pages[kSubs];
                bool ok = true;
#pragma unroll
                for (int sub = 0; sub < kSubs; ++sub) {
                    pages[sub] = sub < nsub ? page_id(a, b, tok0 / kPage + sub) : 0;
                    if (sub < nsub && !page_ok(a, pages[sub]))
                        ok = false;
                }
                if (!ok) {
                    if (slot == 0)
                        raise_error(a.err, KVATTN_DEVERR_PAGE_OUT_OF_RANGE);
                    mbar_arrive(&S.full[st]);
                    continue;
                }
                mbar_arrive_expect_tx(&S.full[st], (uint32_t)(nsub * NKB * kSubRows * 128));
                const int off = tok0 % kPage;
#pragma unroll
                for (int sub = 0; sub < kSubs; ++sub) {
                    if (sub >= nsub)
                        break;
                    const int y = (int)(pages[sub] * kPage) + off;
                    for (int p = 0; p < NKB; ++p) {
                        const int kb = key_box(p);
                        const int col = kb < NVB ? unit_col0 + 64 * kb : a.NU * a.dn + 64 * (kb - NVB);
                        tma_load_2d(S.kv[st] + p * kBoxBytes + sub * kSubRows * 128, &kv_map, col, y, &S.full[st]);
                    }
                }
            }
            // every copy this thread started has landed before the CTA can exit
            for (int st = 0; st < STAGES && st < issued; ++st) {
                const int jl = st + ((issued - 1 - st) / STAGES) * STAGES;
                if (!mbar_wait(&S.full[st], (jl / STAGES) & 1))
                    raise_error(a.err, KVATTN_DEVERR_WAIT_TIMEOUT);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA
        const uint32_t qbase = smem_u32(&S.q[0][0]);
        bool ok = __all_sync(0xffffffffu, mbar_wait(&S.q_ready, 0));
        tc_fence_after();
        // zero rows [ntok, T) of stage st once its copies (whole boxes, rows
        // past the context included) have landed; every lane observes the
        // completed phase before it writes.  False (nothing written) if a
        // lane's wait ran out.
        auto zero_tail = [&](int st, int ntok, uint32_t parity) -> bool {
            if (ntok >= T)
                return true;
            if (!__all_sync(0xffffffffu, mbar_wait(&S.full[st], parity)))
                return false;
            const int rows = T - ntok;
            for (int idx = lane; idx < rows * NKB * 8; idx += 32) {
                const int box = idx / (rows * 8), rem = idx % (rows * 8);
                const int row = ntok + rem / 8, piece = rem % 8;
                *reinterpret_cast<uint4 *>(S.kv[st] + box * kBoxBytes + row * 128 + piece * 16) =
                    make_uint4(0, 0, 0, 0);
            }
            fence_proxy_async_smem();
            __syncwarp();
            return true;
        };
        // Descriptors are built once; a byte offset moves the start-address
        // field by offset >> 4 (shared addresses stay below 256 KB, so the
        // 14-bit field never carries).  The issuing thread does a few integer
        // adds per MMA: with narrow score tiles the MMAs are short and the
        // single issuing thread would otherwise set the pace.
        constexpr uint32_t kStageUnits = Smem::kStageBytes >> 4, kBoxUnits = kBoxBytes >> 4;
        const uint64_t kdesc0 = smem_desc(smem_u32(S.kv[0]), 16, 1024, 2);                      // K-major key boxes
        const uint64_t vdesc0 = smem_desc(smem_u32(S.kv[0]) + NE * kBoxBytes, kBoxBytes, 1024, 2);  // MN-major values
        const uint64_t qdesc0 = smem_desc(qbase, 16, 1024, 2);
        // the score MMAs of tile j
        auto issue_s = [&](int j) {
            if (lane == 0) {
                const uint32_t d = tS + (j & 1) * T;
                const uint64_t kd = kdesc0 + (uint64_t)((j % STAGES) * kStageUnits);
#pragma unroll
                for (int p = 0; p < NKB; ++p) {
                    const int kb = key_box(p);
                    if (kb < NQT) {
                        const uint32_t qa = tQ + kb * 32;
#pragma unroll
                        for (int k = 0; k < 4; ++k)
                            umma_ts(d, qa + k * 8, kd + (uint64_t)(p * kBoxUnits + k * 2), kIdescS, (p | k) ? 1u : 0u);
                    } else {
                        const uint64_t qd = qdesc0 + (uint64_t)((kb - NQT) * (kQChunkBytes >> 4));
#pragma unroll
                        for (int k = 0; k < 4; ++k)
                            umma_ss(d, qd + (uint64_t)(k * 2), kd + (uint64_t)(p * kBoxUnits + k * 2), kIdescS,
                                    (p | k) ? 1u : 0u);
                    }
                }
            }
        };
        // P_t V_t into O (P_t is ready); frees tile t's stage
        auto issue_pv = [&](int t) {
            tc_fence_after();
            if (lane == 0) {
                const uint64_t vd = vdesc0 + (uint64_t)((t % STAGES) * kStageUnits);
                const uint32_t pa = tS + (t & 1) * T;
#pragma unroll
                for (int k = 0; k < T / 16; ++k)
                    umma_ts(tO, pa + 8 * k, vd + (uint64_t)(k * 128), kIdescPV, (t > 0 || k > 0) ? 1u : 0u);
                umma_commit(&S.o_ready);
                umma_commit(&S.empty[t % STAGES]);
            }
            __syncwarp();
        };
        // S_j as soon as its stage is in, then P_{j-1} V_{j-1}
        for (int j = 0; ok && j < n; ++j) {
            const int st = j % STAGES;
            const uint32_t fph = (j / STAGES) & 1;
            if (!__all_sync(0xffffffffu, mbar_wait(&S.full[st], fph))) {
                ok = false;
                break;
            }
            if (!zero_tail(st, tile_ntok<T>(S.pvalid, L, p0, j), fph)) {
                ok = false;
                break;
            }
            tc_fence_after();
            issue_s(j);
            if (lane == 0)
                umma_commit(&S.s_full[j & 1]);
            __syncwarp();
            if (j >= 1) {
                if (!__all_sync(0xffffffffu, mbar_wait(&S.p_full[(j - 1) & 1], ((j - 1) >> 1) & 1)))
                    ok = false;
                else
                    issue_pv(j - 1);
            }
        }
        if (ok && n > 0) {
            if (__all_sync(0xffffffffu, mbar_wait(&S.p_full[(n - 1) & 1], ((n - 1) >> 1) & 1)))
                issue_pv(n - 1);
            else
                ok = false;
        }
        if (!ok && lane == 0)
            raise_error(a.err, KVATTN_DEVERR_WAIT_TIMEOUT);
        // every MMA this thread issued has completed before TMEM is freed
        if (lane == 0)
            umma_commit(&S.mma_done);
        __syncwarp();
        if (!mbar_wait(&S.mma_done, 0) && lane == 0)
            raise_error(a.err, KVATTN_DEVERR_WAIT_TIMEOUT);
        __syncwarp();
    } else {
        // ------------------------------------------------------------ softmax
        constexpr int TH = T / 2;                                // score columns per thread
        constexpr int OH = kDvSlot / 2;                          // output columns per thread
        const int sw = warp - 2;                                 // 0..7
        const int quarter = warp & 3;
        const int half = sw >> 2;                                // column half
        const int h = quarter * 32 + lane;                       // head row = TMEM lane
        const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
        const int rows_used = a.mlra ? a.H : a.HPU;             // GLA: the group's heads
        {
            // validity of every page of this part (read by the MMA warp and here)
            const int npg = min(a.pages_per_split, max(0, (L + kPage - 1) / kPage - p0));
            for (int w = threadIdx.x - 64; w < (npg + 31) / 32; w += kSoftmaxThreads) {
                uint32_t bits = 0;
                for (int i = 32 * w; i < min(npg, 32 * w + 32); ++i)
                    bits |= (page_ok(a, page_id(a, b, p0 + i)) ? 1u : 0u) << (i & 31);
                S.pvalid[w] = bits;
            }
            // Q row h of this slot: [latent query slice | rope query]; chunks
            // below NQT go to TMEM (bf16 pairs), the rest to shared memory;
            // the two threads of a row take alternate chunks
            const __nv_bfloat16 *qn = nullptr, *qr = nullptr;
            if (h < rows_used) {
                size_t row;
                if (a.mlra)
                    row = ((size_t)b * a.H + h) * a.NU + slot;
                else
                    row = (size_t)b * a.H + (size_t)slot * a.HPU + h;
                qn = a.q_nope + row * a.dn;
                qr = a.q_rope + row * a.dr;
            }
#pragma unroll 1
            for (int kb = half; kb < NKB; kb += 2) {
                const __nv_bfloat16 *src = nullptr;
                if (qn)
                    src = kb < NVB ? qn + 64 * kb : qr + 64 * (kb - NVB);
                if (kb < NQT) {
                    uint32_t r[32];
#pragma unroll
                    for (int p = 0; p < 8; ++p) {
                        const uint4 v = src ? *reinterpret_cast<const uint4 *>(src + 8 * p) : make_uint4(0, 0, 0, 0);
                        r[4 * p] = v.x;
                        r[4 * p + 1] = v.y;
                        r[4 * p + 2] = v.z;
                        r[4 * p + 3] = v.w;
                    }
                    tmem_st32(tQ + lane_addr + kb * 32, r);
                } else {
#pragma unroll
                    for (int p = 0; p < 8; ++p) {
                        const uint4 v = src ? *reinterpret_cast<const uint4 *>(src + 8 * p) : make_uint4(0, 0, 0, 0);
                        *reinterpret_cast<uint4 *>(&S.q[kb - NQT][h * 128 + ((p ^ (h & 7)) << 4)]) = v;
                    }
                }
            }
            fence_proxy_async_smem();
            named_sync(1, kSoftmaxThreads);      // page table complete before any role reads it
            tc_fence_before();
            mbar_arrive(&S.q_ready);
        }

        float m_ref = -INFINITY, l = 0.f;       // l: this thread's half of the row sum
        bool ok = true;
        for (int j = 0; j < n; ++j) {
            const int sb = j & 1;
            ok = __all_sync(0xffffffffu, mbar_wait(&S.s_full[sb], (j >> 1) & 1));
            if (!ok)
                break;
            tc_fence_after();
            const uint32_t s_addr = tS + lane_addr + sb * T + half * TH;
            // raw scores: the scale is folded into the exponent's FMA, and the
            // tile maximum of c * s is c times the maximum (for a negative
            // scale the minimum) of the raw scores
            const float c = a.scale_log2;
            float s[TH];
            {
                uint32_t r[TH];
                if constexpr (TH == 64)
                    tmem_ld64(s_addr, r);
                else if constexpr (TH == 32)
                    tmem_ld32(s_addr, r);
                else
                    tmem_ld16(s_addr, r);
#pragma unroll
                for (int i = 0; i < TH; ++i)
                    s[i] = __uint_as_float(r[i]);
            }
            const int ntok = tile_ntok<T>(S.pvalid, L, p0, j);
            const int nvalid = ntok - half * TH;                 // valid columns of this thread
            const bool partial = nvalid < TH;
            float mt;
            if (c >= 0.f) {
                if (partial) {
#pragma unroll
                    for (int i = 0; i < TH; ++i)
                        s[i] = i < nvalid ? s[i] : -INFINITY;
                }
                const float e = reduce_extreme<true, TH>(s);
                mt = e == -INFINITY ? -INFINITY : c * e;
            } else {
                if (partial) {
#pragma unroll
                    for (int i = 0; i < TH; ++i)
                        s[i] = i < nvalid ? s[i] : INFINITY;
                }
                const float e = reduce_extreme<false, TH>(s);
                mt = e == INFINITY ? -INFINITY : c * e;
            }
            // the row max over both halves: swap through shared memory with the
            // partner warp (bounded wait on the quarter's exchange barrier)
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
            const float nm = m_ref == -INFINITY ? 0.f : -m_ref;
            float sx[4] = {0.f, 0.f, 0.f, 0.f}, sy[4] = {0.f, 0.f, 0.f, 0.f};
            uint32_t pk[TH / 2];
#pragma unroll
            for (int i = 0; i < TH / 2; ++i) {
                float x0, x1;
                ffma2(x0, x1, s[2 * i], s[2 * i + 1], c, c, nm, nm);
                if (partial) {
                    x0 = 2 * i < nvalid ? x0 : -INFINITY;
                    x1 = 2 * i + 1 < nvalid ? x1 : -INFINITY;
                }
                const float e0 = exp2_approx(x0), e1 = exp2_approx(x1);
                fadd2(sx[i & 3], sy[i & 3], sx[i & 3], sy[i & 3], e0, e1);
                const __nv_bfloat162 v2 = __floats2bfloat162_rn(e0, e1);
                pk[i] = *reinterpret_cast<const uint32_t *>(&v2);
            }
            const float ps = ((sx[0] + sy[0]) + (sx[1] + sy[1])) + ((sx[2] + sy[2]) + (sx[3] + sy[3]));
            l = l * alpha + ps;
            // P (bf16 pairs) over this half's columns of the score buffer
            const uint32_t p_addr = tS + lane_addr + sb * T + half * (TH / 2);
            if constexpr (TH / 2 == 32)
                tmem_st32(p_addr, pk);
            else if constexpr (TH / 2 == 16)
                tmem_st16(p_addr, pk);
            else
                tmem_st8(p_addr, pk);
            // TMEM accesses are warp-wide: rescale the warp's rows when any needs it
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

        // part result: O / l and lse for this row (l = sum of both halves,
        // swapped in the exchange slot after the last tile's)
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
        const bool valid = h < rows_used;
        const int hu = a.mlra ? h * a.NU + slot : slot * a.HPU + h;
        const size_t prow = ((size_t)b * a.num_splits + split) * a.HU + (valid ? hu : 0);
        float *dst = a.po + prow * a.dn + half * OH;
        const float inv = (have && l > 0.f) ? 1.f / l : 0.f;
        constexpr int CH = OH < 64 ? OH : 64;                     // columns per TMEM load
        uint32_t r[CH];
#pragma unroll 1
        for (int c = 0; c < OH / CH; ++c) {
            if (have) {
                if constexpr (CH == 64)
                    tmem_ld64(tO + lane_addr + half * OH + CH * c, r);
                else
                    tmem_ld32(tO + lane_addr + half * OH + CH * c, r);
            }
            if (valid) {
#pragma unroll
                for (int i = 0; i < CH; i += 4) {
                    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
                    if (have)
                        v = make_float4(__uint_as_float(r[i]) * inv, __uint_as_float(r[i + 1]) * inv,
                                        __uint_as_float(r[i + 2]) * inv, __uint_as_float(r[i + 3]) * inv);
                    *reinterpret_cast<float4 *>(dst + CH * c + i) = v;
                }
            }
        }
        if (valid && half == 0)
            a.plse[prow] = (have && l > 0.f) ? (m_ref + log2f(l)) * kLn2 : -INFINITY;
    }
    __syncwarp();

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0)
        tmem_dealloc(tbase, kTmemCols);
}

template <int T, int NKB, int NVB, int STAGES, int NQT>
cudaError_t launch_latent(const DecodeArgs &a, int slots, cudaStream_t st)
{
    CUtensorMap map;
    const cuuint64_t dims[2] = {(cuuint64_t)a.row, (cuuint64_t)a.num_pages * kPage};
    const cuuint64_t strides[1] = {(cuuint64_t)a.row * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)(T < kPage ? T : kPage)};
    if (encode_tiled(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<__nv_bfloat16 *>(a.kv), dims, strides,
                     box, CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    const size_t smem = sizeof(LatentSmem<T, NKB, STAGES, NQT>);
    auto kern = latent_tc_decode_kernel<T, NKB, NVB, STAGES, NQT>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess)
        return e;
    kern<<<dim3(a.num_splits, slots, a.B), kThreads, smem, st>>>(map, a);
    return cudaGetLastError();
}

}  // namespace

// Shapes the tensor-core latent kernel covers: GLA or MLRA (any number of
// groups or branches, one of them included) with latent slices of 64, 128 or
// 256 columns and a 64-wide rope key; at most 128 query heads per MMA.  Pages
// per part must be a whole number of tiles and fit the validity table.
int latent_tc_page_multiple(const Problem &pr) { return pr.dn <= 128 ? 2 : 1; }
int latent_tc_max_pages_per_split() { return kMaxSplitPages; }

int latent_tc_slots(const Problem &pr)
{
    if (!pr.latent || pr.dr != 64 || (pr.variant != KVATTN_GLA && !pr.mlra))
        return 0;
    if (pr.dn != 64 && pr.dn != 128 && pr.dn != 256)
        return 0;
    return (pr.mlra ? pr.H : pr.HPU) <= kRows ? pr.NU : 0;
}

cudaError_t launch_latent_tc(const DecodeArgs &a, const Problem &pr, cudaStream_t st)
{
    const int slots = latent_tc_slots(pr);
    // <tokens per tile, key boxes, value boxes, stages, Q chunks in TMEM>;
    // TMEM columns 2 T + 64 value boxes + 32 Q chunks stay within 512
    if (pr.dn == 64)
        return launch_latent<128, 2, 1, 4, 2>(a, slots, st);
    if (pr.dn == 128)
        return launch_latent<128, 3, 2, 4, 3>(a, slots, st);
    return launch_latent<64, 5, 4, 4, 4>(a, slots, st);
}

}  // namespace kvattn
