// Absorbed MLA decode on a pair of CTAs: no score is computed twice, and the
// pair's shared memory holds each cached byte once.
//
// After absorption every query head scores the same 576-wide cached row
// [512-d latent | 64-d rope key] and the values are the latent itself (MLRA
// page, MLA paragraph: decode becomes one 576-wide MQA head; MLA explainer
// sections 2.2-2.3).  The scores are a [128 heads x 576] x [576 x tokens]
// contraction and P.V a [128 x tokens] x [tokens x 512] one, so both run as
// tcgen05 MMAs with fp32 accumulators in TMEM.  A 128 x 512 fp32 output fills
// all 512 TMEM columns, so one CTA cannot hold it next to its scores.
//
// The two CTAs of a cluster share one (part, sequence).  CTA r keeps value
// half r (256 columns of O) and, of every 64-token page, scores its own 32
// tokens (rows 32r .. 32r+31) against the whole 576-wide key:
//   * S_r = Q K_own^T            128 x 32, K = 576 (36 MMAs)
//   * row maxima of both token halves swapped with st.async stores that
//     count their bytes on the partner's barrier, so both CTAs follow the
//     same running maximum (and make the same rescale decisions)
//   * P_own (bf16) to this CTA's TMEM, and with st.async stores into one of
//     two buffers in the partner's shared memory (page parity), counted on
//     the partner's barrier; a bulk copy would queue behind the page loads
//     on the SM's copy engine
//   * O_r += [P_0 | P_1] V_r     the page's 64 tokens against this CTA's 256
//     value columns (4 MMAs of N = 256: own P from TMEM, the partner's P from
//     shared memory)
// so the pair issues exactly the algorithmic MMA work.  Each CTA reads its own
// tokens' rows and its value half of the partner's tokens: the page crosses
// HBM once, the shared half is an L2 hit for the later CTA.
//
// A tcgen05.mma with M = 128, K = 16 occupies the tensor pipe for about 47
// cycles whatever N <= 64 is (measured), so the 36 score MMAs of a page cost
// the same for 32 tokens as for 64; halving the tokens halves the stage
// (52 KB against 72 KB) and keeps three stages in flight.
//
// Shared memory (one CTA per SM): Q chunks not in TMEM 48 KB; two rings, E
// (this CTA's 32 rows of the partner's value half and of the rope key, 5 x 4
// KB, read only by the score MMAs and free again when they complete) two
// deep, and V (the page's 64 rows of this CTA's value half, 4 x 8 KB, rows
// 32r.. of which also serve as the own-half key; free after P.V) three deep;
// two buffers of the partner's P (2 x 8 KB: 128 rows x 32 tokens, 64-byte
// swizzle); the max exchange (4 KB).  A 52 KB page load takes about two pages'
// processing time, and the P.V of page j is issued after the scores of page
// j+1: with one 52 KB ring three deep the next page was still loading when
// the MMA thread reached it, the split rings load two pages ahead in 136 KB.
// TMEM: two 32-column score / P buffers, 256 output columns, six 32-column Q
// chunks.
//
// Warp roles (320 threads):
//   warp 0     TMEM allocation; one thread streams pages into the ring (TMA)
//   warp 1     zeroes value rows past the context (0 * NaN would poison the
//              MMA); one thread issues S_j, then P_{j-1} V_{j-1}
//   warps 2-9  two threads per head row, 16 of the CTA's 32 tokens each:
//              online softmax in fp32 (base 2, lazy rescale: the reference
//              maximum moves only when a score exceeds it by more than 2^8)
// Every wait is bounded; a wait that gives up sets an error bit.  Both CTAs
// meet at a cluster barrier before either exits, so no remote store or
// arrival can reach a CTA that has left.
#include <math.h>

#include <type_traits>

#include "latent_common.cuh"

namespace kvattn {

namespace {

using namespace latent;

constexpr int kHalfTok = 32;                              // tokens a CTA scores per page
constexpr int kNKB = 9;                                   // 64-column key boxes: 8 latent + rope
constexpr int kNVB = 4;                                   // value boxes of one CTA (256 columns)
constexpr int kNE = 5;                                    // E boxes: partner's value half + rope
constexpr int kEStages = 2;
constexpr int kVStages = 3;
constexpr int kNQT = 6;                                   // Q chunks held in TMEM
constexpr int kEBoxBytes = kHalfTok * 128;                // 32 rows x 64 bf16
constexpr int kVBoxBytes = kPage * 128;                   // 64 rows x 64 bf16
constexpr int kEBytes = kNE * kEBoxBytes;                 // 20 KB
constexpr int kVBytes = kNVB * kVBoxBytes;                // 32 KB
constexpr int kPBytes = kRows * kHalfTok * 2;             // P of one CTA: 128 rows x 32 tokens (64-byte rows)
constexpr int kSoftmaxThreads = 256;
constexpr int kThreads = 64 + kSoftmaxThreads;
constexpr int kDvSlot = kNVB * 64;                        // 256 output columns per CTA
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kIdescS = idesc_bf16_f32(kRows, kHalfTok, false, false);
constexpr uint32_t kIdescPV = idesc_bf16_f32(kRows, kDvSlot, false, true);

struct PairSmem {
    unsigned char q[kNKB - kNQT][kQChunkBytes];   // Q chunks kNQT..8 (K-major, 128-byte swizzle)
    unsigned char e[kEStages][kEBytes];
    unsigned char v[kVStages][kVBytes];
    unsigned char pp[2][kPBytes];                 // the partner's P of pages of either parity
    float xch[2][4][kRows];                       // [page parity][own half 0, 1, partner half 0, 1][row]
    uint32_t pvalid[kMaxSplitPages / 32];
    uint64_t e_full[kEStages];
    uint64_t e_empty[kEStages];                   // score MMAs done with the E boxes
    uint64_t v_full[kVStages];
    uint64_t v_empty[kVStages];                   // P.V done with the V boxes
    uint64_t s_full[2];
    uint64_t p_full[2];                           // own P in TMEM (and O rescaled)
    uint64_t pp_full[2];                          // the partner's P landed in pp[parity] (1 arrival + 8 KB)
    uint64_t pv_done[2];                          // P.V of a page of that parity completed in both CTAs
    uint64_t o_ready;
    uint64_t q_ready;
    uint64_t mma_done;
    uint64_t xbar[2][4];                          // [page parity][lane quarter]: 64 arrivals + 256 bytes
    uint32_t tmem_base;
};
static_assert(sizeof(PairSmem) <= 227 * 1024, "shared memory budget");
static_assert(2 * kHalfTok + kDvSlot + kNQT * 32 <= (int)kTmemCols, "TMEM budget");

__global__ void __cluster_dims__(1, 2, 1) __launch_bounds__(kThreads, 1)
    latent_pair_decode_kernel(const __grid_constant__ CUtensorMap kv_map, const DecodeArgs a)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    PairSmem &S = *reinterpret_cast<PairSmem *>(smem_raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int split = blockIdx.x, b = blockIdx.z;
    const int r = (int)cluster_ctarank();        // value half and token half of this CTA
    const uint32_t peer = (uint32_t)(r ^ 1);
    pdl_launch_dependents();
    if (smem_u32(smem_raw) & 1023u) {
        // the 128-byte swizzle atoms need 1024-byte alignment; both CTAs of
        // the pair see the same layout and leave before any cluster barrier
        if (threadIdx.x == 0)
            raise_error(a.err, KVATTN_DEVERR_WAIT_TIMEOUT);
        return;
    }

    const int L = row_context(a, b, threadIdx.x == 0 && split == 0 && r == 0);
    const int p0 = split * a.pages_per_split;
    const int tok_end = min(L, (p0 + a.pages_per_split) * kPage);
    const int n = tok_end > p0 * kPage ? (tok_end - p0 * kPage + kPage - 1) / kPage : 0;   // pages

    if (threadIdx.x == 0) {
        for (int st = 0; st < kEStages; ++st) {
            mbar_init(&S.e_full[st], 1);
            mbar_init(&S.e_empty[st], 1);
        }
        for (int st = 0; st < kVStages; ++st) {
            mbar_init(&S.v_full[st], 1);
            mbar_init(&S.v_empty[st], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&S.s_full[i], 1);
            mbar_init(&S.p_full[i], kSoftmaxThreads);
            mbar_init(&S.pp_full[i], 1);
            mbar_init(&S.pv_done[i], 2);
            for (int q = 0; q < 4; ++q)
                mbar_init(&S.xbar[i][q], 64);
        }
        mbar_init(&S.o_ready, 1);
        mbar_init(&S.q_ready, kSoftmaxThreads);
        mbar_init(&S.mma_done, 1);
        fence_mbar_init();
    }
    if (warp == 0)
        tmem_alloc(&S.tmem_base, kTmemCols);
    tc_fence_before();
    cluster_sync_all();          // both CTAs' barriers exist before any remote access
    tc_fence_after();
    const uint32_t tbase = S.tmem_base;
    const uint32_t tS = tbase;                   // 2 score / P buffers of 32 columns
    const uint32_t tO = tbase + 2 * kHalfTok;    // 256 output columns
    const uint32_t tQ = tO + kDvSlot;            // 6 Q chunks of 32 columns (bf16 pairs)

    if (warp == 0) {
        // ---------------------------------------------------------------- TMA
        if (lane == 0 && n > 0) {
            prefetch_tmap(&kv_map);
            int e_issued = 0, v_issued = 0;
            for (int j = 0; j < n; ++j) {
                const long long page = page_id(a, b, p0 + j);
                const bool pg_ok = page_ok(a, page);
                const int y0 = pg_ok ? (int)(page * kPage) : 0;
                if (!pg_ok && r == 0)
                    raise_error(a.err, KVATTN_DEVERR_PAGE_OUT_OF_RANGE);
                // E: this CTA's rows of the partner's value half and of the rope key
                const int es = j % kEStages;
                if (j >= kEStages && !mbar_wait(&S.e_empty[es], ((j / kEStages) - 1) & 1)) {
                    raise_error(a.err, KVATTN_DEVERR_WAIT_TIMEOUT);
                    break;
                }
                e_issued = j + 1;
                if (pg_ok) {
                    mbar_arrive_expect_tx(&S.e_full[es], (uint32_t)kEBytes);
#pragma unroll
                    for (int c = 0; c < kNVB; ++c)
                        tma_load_2d(S.e[es] + c * kEBoxBytes, &kv_map, 64 * ((int)peer * kNVB + c), y0 + kHalfTok * r,
                                    &S.e_full[es]);
                    tma_load_2d(S.e[es] + kNVB * kEBoxBytes, &kv_map, 2 * kDvSlot, y0 + kHalfTok * r, &S.e_full[es]);
                } else {
                    mbar_arrive(&S.e_full[es]);       // nothing loaded: the page counts as outside the context
                }
                // V: all 64 rows of this CTA's value half
                const int vs = j % kVStages;
                if (j >= kVStages && !mbar_wait(&S.v_empty[vs], ((j / kVStages) - 1) & 1)) {
                    raise_error(a.err, KVATTN_DEVERR_WAIT_TIMEOUT);
                    break;
                }
                v_issued = j + 1;
                if (pg_ok) {
                    mbar_arrive_expect_tx(&S.v_full[vs], (uint32_t)kVBytes);
#pragma unroll
                    for (int c = 0; c < kNVB; ++c)
#pragma unroll
                        for (int h2 = 0; h2 < 2; ++h2)
                            tma_load_2d(S.v[vs] + c * kVBoxBytes + h2 * kEBoxBytes, &kv_map, 64 * (r * kNVB + c),
                                        y0 + kHalfTok * h2, &S.v_full[vs]);
                } else {
                    mbar_arrive(&S.v_full[vs]);
                }
            }
            // every copy this thread started has landed before the CTA can exit
            for (int st = 0; st < kEStages && st < e_issued; ++st) {
                const int jl = st + ((e_issued - 1 - st) / kEStages) * kEStages;
                if (!mbar_wait(&S.e_full[st], (jl / kEStages) & 1))
                    raise_error(a.err, KVATTN_DEVERR_WAIT_TIMEOUT);
            }
            for (int st = 0; st < kVStages && st < v_issued; ++st) {
                const int jl = st + ((v_issued - 1 - st) / kVStages) * kVStages;
                if (!mbar_wait(&S.v_full[st], (jl / kVStages) & 1))
                    raise_error(a.err, KVATTN_DEVERR_WAIT_TIMEOUT);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA
        bool ok = __all_sync(0xffffffffu, mbar_wait(&S.q_ready, 0));
        tc_fence_after();
        // Descriptors are built once; a byte offset moves the start-address
        // field by offset >> 4 (shared addresses stay below 256 KB, so the
        // 14-bit field never carries).
        const uint64_t edesc0 = smem_desc(smem_u32(S.e[0]), 16, 1024, 2);     // K-major key rows (E)
        const uint64_t kvdesc0 = smem_desc(smem_u32(S.v[0]), 16, 1024, 2);    // K-major key rows (own half)
        const uint64_t vdesc0 = smem_desc(smem_u32(S.v[0]), kVBoxBytes, 1024, 2);   // MN-major values
        const uint64_t qdesc0 = smem_desc(smem_u32(&S.q[0][0]), 16, 1024, 2);
        // the partner's P: K-major, 64-byte rows, 64-byte swizzle (8-row atoms of 512 bytes)
        const uint64_t pdesc0 = smem_desc(smem_u32(S.pp[0]), 16, 512, 4);
        // zero value rows [ntok, 64) of V slot vs (whole 128-byte rows, so
        // the swizzle does not matter); the rows also hold the own-half key
        // rows past the context, whose scores the softmax masks anyway
        auto zero_tail = [&](int vs, int ntok) {
            if (ntok >= kPage)
                return;
            const int rows = kPage - ntok;
            for (int idx = lane; idx < rows * 8 * kNVB; idx += 32) {
                const int box = idx / (rows * 8), rem = idx % (rows * 8);
                const int row = ntok + rem / 8, piece = rem % 8;
                *reinterpret_cast<uint4 *>(S.v[vs] + box * kVBoxBytes + row * 128 + piece * 16) =
                    make_uint4(0, 0, 0, 0);
            }
            fence_proxy_async_smem();
            __syncwarp();
        };
        // the score MMAs of page j, in one fully unrolled copy per rank: the
        // box sources and offsets are constants, so each MMA issues with no
        // address work (the issuing thread otherwise sets the pace)
        auto issue_s_rank = [&](auto rank, int j) {
            constexpr int R = decltype(rank)::value;
            const uint32_t d = tS + (j & 1) * kHalfTok;
            const uint64_t ed = edesc0 + (uint64_t)((j % kEStages) * (kEBytes >> 4));
            const uint64_t vd = kvdesc0 + (uint64_t)((j % kVStages) * (kVBytes >> 4));
#pragma unroll
            for (int kb = 0; kb < kNKB; ++kb) {
                const bool in_v = kb < kNKB - 1 && kb / kNVB == R;
                const uint32_t off = (kb == kNKB - 1 ? kNVB * kEBoxBytes
                                      : in_v       ? (kb % kNVB) * kVBoxBytes + R * kEBoxBytes
                                                   : (kb % kNVB) * kEBoxBytes) >> 4;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const uint64_t bd = (in_v ? vd : ed) + (uint64_t)(off + k * 2);
                    const uint32_t acc = (kb | k) ? 1u : 0u;
                    if (kb < kNQT)
                        umma_ts(d, tQ + kb * 32 + k * 8, bd, kIdescS, acc);
                    else
                        umma_ss(d, qdesc0 + (uint64_t)((kb - kNQT) * (kQChunkBytes >> 4) + k * 2), bd, kIdescS, acc);
                }
            }
        };
        auto issue_s = [&](int j) {
            if (lane == 0) {
                if (r == 0)
                    issue_s_rank(std::integral_constant<int, 0>{}, j);
                else
                    issue_s_rank(std::integral_constant<int, 1>{}, j);
                umma_commit(&S.s_full[j & 1]);
                umma_commit(&S.e_empty[j % kEStages]);
            }
            __syncwarp();
        };
        // O += [P_0 | P_1] V over the page's 64 tokens (16 per MMA): the
        // tokens of half r come from this CTA's TMEM, the others from the
        // partner's P in shared memory
        // P.V of page t, one copy per rank: the 16-token steps of this CTA's
        // half read P from TMEM, the partner's half from shared memory
        auto issue_pv_rank = [&](auto rank, int t) {
            constexpr int R = decltype(rank)::value;
            const uint64_t vd = vdesc0 + (uint64_t)((t % kVStages) * (kVBytes >> 4));
            const uint32_t pa = tS + (t & 1) * kHalfTok;
            const uint64_t pd = pdesc0 + (uint64_t)((t & 1) * (kPBytes >> 4));
#pragma unroll
            for (int s = 0; s < 4; ++s) {
                const uint32_t acc = (t > 0 || s > 0) ? 1u : 0u;
                if ((s >> 1) == R)
                    umma_ts(tO, pa + 8 * (s & 1), vd + (uint64_t)(s * 128), kIdescPV, acc);
                else
                    umma_ss(tO, pd + (uint64_t)((s & 1) * 2), vd + (uint64_t)(s * 128), kIdescPV, acc);
            }
        };
        auto issue_pv = [&](int t) {
            tc_fence_after();
            if (lane == 0) {
                if (r == 0)
                    issue_pv_rank(std::integral_constant<int, 0>{}, t);
                else
                    issue_pv_rank(std::integral_constant<int, 1>{}, t);
                umma_commit(&S.o_ready);
                umma_commit(&S.v_empty[t % kVStages]);
                umma_commit_multicast(&S.pv_done[t & 1], 0x3);
            }
            __syncwarp();
        };
        // the partner's P of pages 0 and 1 may land from now on
        if (lane == 0) {
            for (int t = 0; t < 2 && t < n; ++t)
                mbar_arrive_expect_tx(&S.pp_full[t], (uint32_t)kPBytes);
        }
        for (int j = 0; ok && j <= n; ++j) {
            if (j < n) {
                const int es = j % kEStages, vs = j % kVStages;
                const int ntok = tile_ntok<kPage>(S.pvalid, L, p0, j);
                const bool in =
                    mbar_wait(&S.v_full[vs], (j / kVStages) & 1) && mbar_wait(&S.e_full[es], (j / kEStages) & 1);
                if (!__all_sync(0xffffffffu, in)) {
                    ok = false;
                    break;
                }
                zero_tail(vs, ntok);
                tc_fence_after();
                issue_s(j);
            }
            if (j >= 1) {
                const int t = j - 1;
                const bool in =
                    mbar_wait(&S.p_full[t & 1], (t >> 1) & 1) && mbar_wait(&S.pp_full[t & 1], (t >> 1) & 1);
                if (!__all_sync(0xffffffffu, in)) {
                    ok = false;
                    break;
                }
                if (lane == 0) {
                    // the partner's P arrived as generic-proxy stores: order
                    // them before the MMA's (async-proxy) reads
                    fence_proxy_async_smem();
                    // arm the buffer for page t + 2's P before this page's
                    // P.V can release the partner to send it
                    if (t + 2 < n)
                        mbar_arrive_expect_tx(&S.pp_full[t & 1], (uint32_t)kPBytes);
                }
                issue_pv(t);
            }
        }
        if (!ok && lane == 0)
            raise_error(a.err, KVATTN_DEVERR_WAIT_TIMEOUT);
        // every MMA this thread issued has completed before TMEM is freed, and
        // both CTAs' P.V arrivals for the last pages have reached this CTA
        if (lane == 0)
            umma_commit(&S.mma_done);
        __syncwarp();
        bool drained = mbar_wait(&S.mma_done, 0);
        if (ok && n > 0) {
            for (int t = max(0, n - 2); t < n; ++t)
                drained = mbar_wait_cluster(&S.pv_done[t & 1], (t >> 1) & 1) && drained;
        }
        if (!drained && lane == 0)
            raise_error(a.err, KVATTN_DEVERR_WAIT_TIMEOUT);
        __syncwarp();
    } else {
        // ------------------------------------------------------------ softmax
        const int sw = warp - 2;                                 // 0..7
        const int quarter = warp & 3;
        const int half = sw >> 2;                                // which 16 of the CTA's 32 tokens
        const int h = quarter * 32 + lane;                       // head row = TMEM lane
        const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
        const uint32_t peer_xch = mapa_shared(smem_u32(&S.xch[0][0][0]), peer);
        const uint32_t peer_xbar0 = mapa_shared(smem_u32(&S.xbar[0][quarter]), peer);
        const uint32_t peer_xbar1 = mapa_shared(smem_u32(&S.xbar[1][quarter]), peer);
        const uint32_t peer_pp = mapa_shared(smem_u32(S.pp[0]), peer);
        const uint32_t peer_pp_full = mapa_shared(smem_u32(&S.pp_full[0]), peer);
        const bool arm = half == 0 && lane == 0;                 // carries the partner's 256 bytes
        {
            // validity of every page of this part (read by the MMA warp and here)
            const int npg = min(a.pages_per_split, max(0, (L + kPage - 1) / kPage - p0));
            fill_page_bits(S.pvalid, a, b, p0, npg, threadIdx.x - 64, kSoftmaxThreads);
            // Q row h as key boxes [latent 0..7 | rope]; chunks below kNQT go
            // to TMEM (bf16 pairs), the rest to shared memory; the two threads
            // of a row take alternate chunks
            const bool row_on = h < a.H;
#pragma unroll 1
            for (int kb = half; kb < kNKB; kb += 2) {
                const __nv_bfloat16 *src = nullptr;
                if (row_on)
                    src = kb == kNKB - 1 ? a.q_rope + ((size_t)b * a.H + h) * a.dr
                                         : a.q_nope + ((size_t)b * a.H + h) * a.dn + 64 * kb;
                uint4 v[8];
#pragma unroll
                for (int p = 0; p < 8; ++p)
                    v[p] = src ? *reinterpret_cast<const uint4 *>(src + 8 * p) : make_uint4(0, 0, 0, 0);
                if (kb < kNQT) {
                    uint32_t rr[32];
#pragma unroll
                    for (int p = 0; p < 8; ++p) {
                        rr[4 * p] = v[p].x;
                        rr[4 * p + 1] = v[p].y;
                        rr[4 * p + 2] = v[p].z;
                        rr[4 * p + 3] = v[p].w;
                    }
                    tmem_st32(tQ + lane_addr + kb * 32, rr);
                } else {
#pragma unroll
                    for (int p = 0; p < 8; ++p)
                        *reinterpret_cast<uint4 *>(&S.q[kb - kNQT][h * 128 + ((p ^ (h & 7)) << 4)]) = v[p];
                }
            }
            fence_proxy_async_smem();
            named_sync(1, kSoftmaxThreads);      // page table complete before any role reads it
            tc_fence_before();
            mbar_arrive(&S.q_ready);
        }

        // the row maximum (or sum) over the page's four 16-token quarters: the
        // partner thread of this CTA through shared memory, the other CTA's
        // two threads through st.async stores counted on this quarter's barrier
        auto exchange = [&](int j, float v, float *o) -> bool {
            const int sb = j & 1;
            S.xch[sb][half][h] = v;
            st_async_f32(peer_xch + (uint32_t)(((sb * 4 + 2 + half) * kRows + h) * 4), v,
                         sb ? peer_xbar1 : peer_xbar0);
            if (arm)
                mbar_arrive_expect_tx(&S.xbar[sb][quarter], 64 * 4);
            else
                mbar_arrive(&S.xbar[sb][quarter]);
            if (!__all_sync(0xffffffffu, mbar_wait_cluster(&S.xbar[sb][quarter], (j >> 1) & 1)))
                return false;
            o[0] = S.xch[sb][0][h];
            o[1] = S.xch[sb][1][h];
            o[2] = S.xch[sb][2][h];
            o[3] = S.xch[sb][3][h];
            return true;
        };

        float m_ref = -INFINITY, l = 0.f;       // l: this thread's 16 tokens of every page
        bool ok = true;
        for (int j = 0; j < n; ++j) {
            const int sb = j & 1;
            ok = __all_sync(0xffffffffu, mbar_wait(&S.s_full[sb], (j >> 1) & 1));
            if (!ok)
                break;
            tc_fence_after();
            float s[16];
            {
                uint32_t rr[16];
                tmem_ld16(tS + lane_addr + sb * kHalfTok + half * 16, rr);
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    s[i] = __uint_as_float(rr[i]) * a.scale_log2;
            }
            const int ntok = tile_ntok<kPage>(S.pvalid, L, p0, j);
            const int own = min(max(ntok - kHalfTok * r, 0), kHalfTok) - half * 16;   // valid of my 16
            if (own < 16) {
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    s[i] = i < own ? s[i] : -INFINITY;
            }
            float mt = fmaxf(fmaxf(fmaxf(s[0], s[1]), fmaxf(s[2], s[3])), fmaxf(fmaxf(s[4], s[5]), fmaxf(s[6], s[7])));
            mt = fmaxf(mt, fmaxf(fmaxf(fmaxf(s[8], s[9]), fmaxf(s[10], s[11])),
                                 fmaxf(fmaxf(s[12], s[13]), fmaxf(s[14], s[15]))));
            float x4[4];
            ok = exchange(j, mt, x4);
            if (!ok)
                break;
            mt = fmaxf(fmaxf(x4[0], x4[1]), fmaxf(x4[2], x4[3]));

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
            uint32_t pk[8];
            float ps0 = 0.f, ps1 = 0.f;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float e0 = exp2_approx(s[2 * i] - m_use), e1 = exp2_approx(s[2 * i + 1] - m_use);
                ps0 += e0;
                ps1 += e1;
                const __nv_bfloat162 v2 = __floats2bfloat162_rn(e0, e1);
                pk[i] = *reinterpret_cast<const uint32_t *>(&v2);
            }
            l = l * alpha + (ps0 + ps1);
            // own P into the partner's buffer of this page's parity, once the
            // partner's P.V of page j-2 has read it: row h of 64 bytes,
            // tokens 16*half .. 16*half+15 as two 16-byte chunks, chunk c
            // stored at c ^ ((h >> 1) & 3) (64-byte swizzle)
            if (j >= 2) {
                ok = __all_sync(0xffffffffu, mbar_wait_cluster(&S.pv_done[sb], ((j - 2) >> 1) & 1));
                if (!ok)
                    break;
            }
            {
                const uint32_t row = peer_pp + (uint32_t)(sb * kPBytes + h * (kHalfTok * 2));
                const uint32_t bar = peer_pp_full + (uint32_t)(sb * 8);
                const uint32_t c0 = (uint32_t)(2 * half), sw4 = (uint32_t)((h >> 1) & 3);
                st_async_u32x4(row + ((c0 ^ sw4) << 4), pk[0], pk[1], pk[2], pk[3], bar);
                st_async_u32x4(row + (((c0 + 1) ^ sw4) << 4), pk[4], pk[5], pk[6], pk[7], bar);
            }
            // own P into the score buffer it came from (A operand of this
            // CTA's P.V); S_j has completed, so P_{j-2} there is consumed
            tmem_st8(tS + lane_addr + sb * kHalfTok + half * 8, pk);
            // TMEM accesses are warp-wide: rescale the warp's rows when any needs it
            if (__any_sync(0xffffffffu, rescale)) {
                ok = __all_sync(0xffffffffu, mbar_wait(&S.o_ready, (j - 1) & 1));
                if (!ok)
                    break;
                tc_fence_after();
                uint32_t rr[32];
#pragma unroll 1
                for (int c = 0; c < kDvSlot / 2 / 32; ++c) {
                    const uint32_t o_addr = tO + lane_addr + half * (kDvSlot / 2) + 32 * c;
                    tmem_ld32(o_addr, rr);
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        rr[i] = __float_as_uint(__uint_as_float(rr[i]) * alpha);
                    tmem_st32(o_addr, rr);
                }
            }
            tc_fence_before();
            mbar_arrive(&S.p_full[sb]);
        }
        if (!ok && lane == 0)
            raise_error(a.err, KVATTN_DEVERR_WAIT_TIMEOUT);

        // part result: O / l and lse for this row, l summed over the four
        // token quarters through the same exchange
        if (ok) {
            float x4[4];
            ok = exchange(n, l, x4);
            if (ok)
                l = (x4[0] + x4[1]) + (x4[2] + x4[3]);
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
        // value columns [256r, 256r + 256) of every row
        const bool valid = h < a.H;
        const size_t prow = ((size_t)b * a.num_splits + split) * a.HU + (valid ? h : 0);
        float *dst = a.po + prow * a.dn + r * kDvSlot + half * (kDvSlot / 2);
        const float inv = (have && l > 0.f) ? 1.f / l : 0.f;
        uint32_t rr[64];
#pragma unroll 1
        for (int c = 0; c < kDvSlot / 2 / 64; ++c) {
            if (have)
                tmem_ld64(tO + lane_addr + half * (kDvSlot / 2) + 64 * c, rr);
            if (valid) {
#pragma unroll
                for (int i = 0; i < 64; i += 4) {
                    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
                    if (have)
                        v = make_float4(__uint_as_float(rr[i]) * inv, __uint_as_float(rr[i + 1]) * inv,
                                        __uint_as_float(rr[i + 2]) * inv, __uint_as_float(rr[i + 3]) * inv);
                    *reinterpret_cast<float4 *>(dst + 64 * c + i) = v;
                }
            }
        }
        if (valid && half == 0 && r == 0)
            a.plse[prow] = (have && l > 0.f) ? (m_ref + log2f(l)) * kLn2 : -INFINITY;
    }
    __syncwarp();

    tc_fence_before();
    cluster_sync_all();          // no remote store, copy or arrival is still headed for either CTA
    tc_fence_after();
    if (warp == 0)
        tmem_dealloc(tbase, kTmemCols);
}

}  // namespace

// Absorbed MLA: one 512-wide latent + 64-wide rope key, at most 128 heads.
bool latent_pair_supported(const Problem &pr)
{
    return pr.latent && !pr.mlra && pr.NU == 1 && pr.dn == 512 && pr.dr == 64 && pr.H <= kRows;
}

cudaError_t launch_latent_pair(const DecodeArgs &a, cudaStream_t st)
{
    CUtensorMap map;
    const cuuint64_t dims[2] = {(cuuint64_t)a.row, (cuuint64_t)a.num_pages * kPage};
    const cuuint64_t strides[1] = {(cuuint64_t)a.row * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)kHalfTok};
    if (encode_tiled(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<__nv_bfloat16 *>(a.kv), dims, strides,
                     box, CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    const size_t smem = sizeof(PairSmem);
    cudaError_t e =
        cudaFuncSetAttribute(latent_pair_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess)
        return e;
    latent_pair_decode_kernel<<<dim3(a.num_splits, 2, a.B), kThreads, smem, st>>>(map, a);
    return cudaGetLastError();
}

}  // namespace kvattn
