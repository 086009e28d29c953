// Host side of the C ABI declared in include/kvattn.h: argument validation,
// launch planning, workspace layout and the two launches of one decode call.
// Nothing here allocates device memory or reads it back, except
// kvattn_get_device_error.
#include <math.h>
#include <string.h>

#include "kvattn_internal.cuh"

namespace kvattn {

// The GQA kernel over an fp8 (e4m3) cache (decode_gqa_fp8.cu).
bool gqa_fp8_supported(const Problem &pr);
cudaError_t launch_gqa_fp8(const DecodeArgs &a, float k_scale, float v_scale, cudaStream_t st);
namespace {

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

constexpr int kMaxDevices = 64;

int validate(int32_t variant, const kvattn_params *p, Problem *pr)
{
    if (!p || !pr)
        return KVATTN_ERR_INVALID_ARG;
    if (variant < KVATTN_GQA || variant > KVATTN_GTA)
        return KVATTN_ERR_UNSUPPORTED;
    if (p->batch < 1 || p->num_q_heads < 1 || p->num_kv < 1 || p->d_nope < 1 || p->d_rope < 0 ||
        p->max_pages_per_seq < 1 || p->num_pages < 1 || p->max_seq_len < 0 || p->num_splits < 0)
        return KVATTN_ERR_INVALID_ARG;
    if (p->out_dtype != KVATTN_OUT_BF16 && p->out_dtype != KVATTN_OUT_FP32)
        return KVATTN_ERR_INVALID_ARG;
    if (p->q_len < 0)
        return KVATTN_ERR_INVALID_ARG;
    if (p->branch_out != 0 && (p->branch_out != 1 || variant != KVATTN_MLRA))
        return KVATTN_ERR_INVALID_ARG;
    if (p->cache_dtype != KVATTN_CACHE_BF16 && p->cache_dtype != KVATTN_CACHE_FP8_E4M3)
        return KVATTN_ERR_INVALID_ARG;
    if (p->cache_dtype == KVATTN_CACHE_FP8_E4M3) {
        if (!(p->k_scale > 0.f) || !(p->v_scale > 0.f) || !isfinite(p->k_scale) || !isfinite(p->v_scale))
            return KVATTN_ERR_INVALID_ARG;
        if (variant != KVATTN_GQA)
            return KVATTN_ERR_UNSUPPORTED;
    }
    const int q_len = p->q_len > 0 ? p->q_len : 1;
    if (q_len > kMaxQueryLen || (long long)p->batch * q_len > 65535 || p->num_q_heads > 65535)
        return KVATTN_ERR_UNSUPPORTED;
    if (p->page_size != kPage)
        return KVATTN_ERR_UNSUPPORTED;
    if ((long long)p->max_seq_len > (long long)p->max_pages_per_seq * kPage)
        return KVATTN_ERR_INVALID_ARG;
    if (p->d_nope % 8 || p->d_rope % 8)
        return KVATTN_ERR_UNSUPPORTED;
    if (p->d_nope > 512 || p->d_rope > 128)
        return KVATTN_ERR_UNSUPPORTED;
    const bool latent = variant == KVATTN_MLA || variant == KVATTN_GLA || variant == KVATTN_MLRA;
    if (!latent && p->d_rope != 0)
        return KVATTN_ERR_INVALID_ARG;
    if ((variant == KVATTN_MQA || variant == KVATTN_MLA) && p->num_kv != 1)
        return KVATTN_ERR_INVALID_ARG;
    if ((variant == KVATTN_GQA || variant == KVATTN_GLA || variant == KVATTN_GTA) && p->num_q_heads % p->num_kv)
        return KVATTN_ERR_INVALID_ARG;
    if (variant == KVATTN_MLRA && p->num_kv > 16)
        return KVATTN_ERR_UNSUPPORTED;
    const long long row = latent ? (long long)p->num_kv * p->d_nope + p->d_rope
                                 : (long long)p->num_kv * p->d_nope;
    if (row > (1 << 20))
        return KVATTN_ERR_UNSUPPORTED;

    pr->variant = variant;
    pr->B = p->batch * q_len;     // one row per (sequence, query position)
    pr->q_len = q_len;
    pr->H = p->num_q_heads;
    pr->NU = p->num_kv;
    pr->dn = p->d_nope;
    pr->dr = p->d_rope;
    pr->Dk = p->d_nope + p->d_rope;
    pr->Dv = p->d_nope;
    pr->row = (int)row;
    pr->latent = latent;
    pr->mlra = variant == KVATTN_MLRA;
    pr->HPU = pr->mlra ? pr->H : pr->H / pr->NU;
    pr->HU = pr->mlra ? pr->H * pr->NU : pr->H;
    pr->mpps = p->max_pages_per_seq;
    pr->num_pages = p->num_pages;
    pr->max_seq_len = p->max_seq_len;
    pr->out_dtype = p->out_dtype;
    pr->paged = true;
    pr->branch_out = p->branch_out != 0;
    pr->kv_planes = variant == KVATTN_GTA ? 1 : 2;
    return KVATTN_OK;
}

// Heads per CTA of the generic kernel: the unit's heads, in chunks of at most 16.
int generic_head_chunk(const Problem &pr)
{
    const int hpu = pr.HPU;
    if (hpu >= 16)
        return hpu % 16 == 0 ? 16 : 0;
    if (hpu == 1 || hpu == 2 || hpu == 4 || hpu == 8)
        return hpu;
    return 0;
}

struct Plan {
    kvattn_plan pub;
    int head_chunk;
    int head_chunks;
    size_t ticket_bytes;  // per (sequence, unit) part counters for in-kernel merges
    size_t lse_bytes;
    bool fused_merge;     // the decode kernel merges its own parts (no combine launch)
};

// Parts per context: forced, or enough CTAs for several waves over the SMs
// (counted from the longest context, the only length the host knows).
int choose_splits(int forced, long long units, int max_pages, long long target_ctas, int min_pages_per_split)
{
    int splits;
    if (forced > 0) {
        splits = forced;
    } else {
        splits = (int)((target_ctas + units - 1) / units);
        const int cap = (max_pages + min_pages_per_split - 1) / min_pages_per_split;
        splits = splits > cap ? cap : splits;
    }
    splits = splits < 1 ? 1 : splits;
    splits = splits > max_pages ? max_pages : splits;
    splits = splits > kMaxSplits ? kMaxSplits : splits;
    return splits;
}

int make_plan(const Problem &pr, int forced_splits, Plan *pl)
{
    memset(pl, 0, sizeof *pl);
    const int num_sms = sm_count();
    const int max_pages = pr.max_seq_len > 0 ? (pr.max_seq_len + kPage - 1) / kPage : 1;
    long long base;
    int splits;
    const bool pair = latent_pair_supported(pr);
    const int tc_slots = pair ? 2 : latent_tc_slots(pr);
    if (tc_slots > 0) {
        pl->pub.kernel = pair ? KVATTN_KERNEL_LATENT_PAIR : KVATTN_KERNEL_LATENT_TC;
        pl->head_chunk = 128;
        pl->head_chunks = tc_slots;
        base = (long long)pr.B * tc_slots;
        // one CTA per SM: for small batches the fewest waves that keep >= 90% of
        // the SMs busy (long parts, little partial-output traffic); several
        // waves to even out ragged large batches
        long long target = 4LL * num_sms;
        if (base < num_sms / 2) {
            for (long long k = 1; k <= 4; ++k) {
                const long long sp = (k * num_sms) / base;
                const long long ctas = sp * base;
                const long long waves = (ctas + num_sms - 1) / num_sms;
                target = ctas;
                if (sp >= 1 && ctas * 10 >= waves * num_sms * 9)
                    break;
            }
        }
        splits = choose_splits(forced_splits, base, max_pages, target, pr.mlra ? 16 : 64);
    } else if (gqa_supported(pr)) {
        pl->pub.kernel = KVATTN_KERNEL_GQA;
        pl->head_chunk = 4;
        pl->head_chunks = 1;
        base = (long long)pr.B * pr.NU;
        splits = choose_splits(forced_splits, base, max_pages, 4LL * 3 * num_sms, 4);
    } else if (mqa_mma_supported(pr)) {
        pl->pub.kernel = KVATTN_KERNEL_MQA_TC;
        pl->head_chunk = 32;
        pl->head_chunks = 1;
        base = (long long)pr.B * pr.NU;
        // about 1.3 waves of one CTA per SM: measured on 32 x U[1024,8192]
        // contexts (decode + combine), 6 parts 48.3 us, 7 parts 49.8, 12 parts
        // 54.3, 8 parts 60.1 (1.7 waves), 4 parts 60.4 (under one wave)
        splits = choose_splits(forced_splits, base, max_pages, 13LL * num_sms / 10, 2);
    } else {
        const int hc = generic_head_chunk(pr);
        if (!hc)
            return KVATTN_ERR_UNSUPPORTED;
        if (generic_smem_bytes(pr, hc) > 227 * 1024)
            return KVATTN_ERR_UNSUPPORTED;
        pl->pub.kernel = KVATTN_KERNEL_GENERIC;
        pl->head_chunk = hc;
        pl->head_chunks = pr.HPU / hc;
        base = (long long)pr.B * pr.NU * pl->head_chunks;
        splits = choose_splits(forced_splits, base, max_pages, 2LL * num_sms, 1);
    }
    int pps = (max_pages + splits - 1) / splits;
    if (pl->pub.kernel == KVATTN_KERNEL_LATENT_TC || pl->pub.kernel == KVATTN_KERNEL_LATENT_PAIR) {
        // whole tiles per part, and no more pages than the kernel's page table holds
        const int m = pl->pub.kernel == KVATTN_KERNEL_LATENT_PAIR ? 1 : latent_tc_page_multiple(pr);
        const int cap = latent_tc_max_pages_per_split();
        pps = (pps + m - 1) / m * m;
        if (pps > cap)
            pps = cap;
    }
    splits = (max_pages + pps - 1) / pps;
    if (splits > kMaxSplits)
        return KVATTN_ERR_UNSUPPORTED;
    pl->pub.num_splits = splits;
    pl->pub.pages_per_split = pps;
    pl->pub.ctas = (int32_t)(base * splits);
    // the GQA kernel merges its own parts (a few KB per group); the MQA and
    // latent groups are hundreds of KB to MB, merged faster by the combine grid
    pl->fused_merge = pl->pub.kernel == KVATTN_KERNEL_GQA;
    pl->pub.launches = pl->fused_merge ? 1 : 2;
    pl->ticket_bytes = align_up((size_t)pr.B * pr.NU * sizeof(int), 256);
    pl->pub.header_bytes = (int32_t)(kWsHeader + pl->ticket_bytes);
    const size_t rows = (size_t)pr.B * splits * pr.HU;
    pl->lse_bytes = align_up(rows * sizeof(float), 256);
    pl->pub.workspace_bytes = kWsHeader + pl->ticket_bytes + pl->lse_bytes + rows * pr.Dv * sizeof(float);
    return KVATTN_OK;
}

// The plan of a call: the cache element type picks the kernel for the same
// geometry (an fp8 cache has its own GQA kernel; other shapes are refused).
int plan_call(const kvattn_params *p, const Problem &pr, Plan *pl)
{
    if (p->cache_dtype == KVATTN_CACHE_FP8_E4M3 && !gqa_fp8_supported(pr))
        return KVATTN_ERR_UNSUPPORTED;
    const int st = make_plan(pr, p->num_splits, pl);
    if (st)
        return st;
    if (p->cache_dtype == KVATTN_CACHE_FP8_E4M3) {
        // same grid, parts and in-kernel merge as the bf16 GQA plan
        if (pl->pub.kernel != KVATTN_KERNEL_GQA || !pl->fused_merge)
            return KVATTN_ERR_UNSUPPORTED;
        pl->pub.kernel = KVATTN_KERNEL_GQA_FP8;
    }
    return KVATTN_OK;
}

}  // namespace

int sm_count()
{
    static int cached[kMaxDevices] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();   // a failed query leaves its error as the last error: clear it
        return kDefaultSMs;
    }
    if (!cached[dev]) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1) {
            cudaGetLastError();
            return kDefaultSMs;
        }
        cached[dev] = n;
    }
    return cached[dev];
}

int validate_params(int32_t variant, const kvattn_params *p, Problem *pr) { return validate(variant, p, pr); }

int validate_call(int32_t variant, const kvattn_params *p, const void *q_nope, const void *q_rope,
                  const void *kv_cache, const int32_t *block_table, const int32_t *seq_lens,
                  float sm_scale, const void *out, const float *lse, const void *workspace,
                  Problem *pr)
{
    int st = validate(variant, p, pr);
    if (st)
        return st;
    if (!q_nope || !kv_cache || !seq_lens || !out || !workspace)
        return KVATTN_ERR_INVALID_ARG;
    if (pr->dr > 0 && !q_rope)
        return KVATTN_ERR_INVALID_ARG;
    if (!isfinite(sm_scale))
        return KVATTN_ERR_INVALID_ARG;
    if (!aligned(q_nope, 16) || (q_rope && !aligned(q_rope, 16)) || !aligned(kv_cache, 16) ||
        !aligned(out, 16) || (lse && !aligned(lse, 4)) || !aligned(workspace, 256) ||
        !aligned(seq_lens, 4) || (block_table && !aligned(block_table, 4)))
        return KVATTN_ERR_MISALIGNED;
    return KVATTN_OK;
}

}  // namespace kvattn

using namespace kvattn;

extern "C" int kvattn_version(void) { return 202; }

extern "C" const char *kvattn_status_string(int status)
{
    switch (status) {
    case KVATTN_OK: return "ok";
    case KVATTN_ERR_INVALID_ARG: return "invalid argument";
    case KVATTN_ERR_UNSUPPORTED: return "unsupported problem";
    case KVATTN_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case KVATTN_ERR_MISALIGNED: return "misaligned pointer";
    case KVATTN_ERR_CUDA: return "CUDA error";
    default: return "unknown status";
    }
}

extern "C" int kvattn_get_plan(int32_t variant, const kvattn_params *p, kvattn_plan *plan)
{
    if (!plan)
        return KVATTN_ERR_INVALID_ARG;
    Problem pr;
    int st = validate(variant, p, &pr);
    if (st)
        return st;
    Plan pl;
    st = plan_call(p, pr, &pl);
    if (st)
        return st;
    *plan = pl.pub;
    return KVATTN_OK;
}

extern "C" int kvattn_workspace_size(int32_t variant, const kvattn_params *p, size_t *bytes)
{
    if (!bytes)
        return KVATTN_ERR_INVALID_ARG;
    kvattn_plan plan;
    const int st = kvattn_get_plan(variant, p, &plan);
    if (st)
        return st;
    *bytes = (size_t)plan.workspace_bytes;
    return KVATTN_OK;
}

extern "C" int kvattn_workspace_init(void *workspace, size_t workspace_bytes, void *stream)
{
    if (!workspace || workspace_bytes < kWsHeader)
        return KVATTN_ERR_INVALID_ARG;
    if (!aligned(workspace, 256))
        return KVATTN_ERR_MISALIGNED;
    if (cudaMemsetAsync(workspace, 0, workspace_bytes, static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return KVATTN_ERR_CUDA;
    return KVATTN_OK;
}

extern "C" int kvattn_decode_timed(int32_t variant, const kvattn_params *p, const void *q_nope,
                                   const void *q_rope, const void *kv_cache,
                                   const int32_t *block_table, const int32_t *seq_lens,
                                   float sm_scale, void *out, float *lse, void *workspace,
                                   size_t workspace_bytes, void *stream, void *const *events)
{
    Problem pr;
    int st = validate_call(variant, p, q_nope, q_rope, kv_cache, block_table, seq_lens, sm_scale, out,
                           lse, workspace, &pr);
    if (st)
        return st;
    Plan pl;
    st = plan_call(p, pr, &pl);
    if (st)
        return st;
    if (workspace_bytes < pl.pub.workspace_bytes)
        return KVATTN_ERR_WORKSPACE_TOO_SMALL;

    char *ws = static_cast<char *>(workspace);
    DecodeArgs a{};
    a.q_nope = static_cast<const __nv_bfloat16 *>(q_nope);
    a.q_rope = static_cast<const __nv_bfloat16 *>(q_rope);
    a.kv = static_cast<const __nv_bfloat16 *>(kv_cache);
    a.block_table = block_table;
    a.seq_lens = seq_lens;
    a.err = reinterpret_cast<int *>(ws);
    a.tickets = reinterpret_cast<int *>(ws + kWsHeader);
    a.plse = reinterpret_cast<float *>(ws + kWsHeader + pl.ticket_bytes);
    a.po = reinterpret_cast<float *>(ws + kWsHeader + pl.ticket_bytes + pl.lse_bytes);
    a.out = out;
    a.lse_out = lse;
    a.out_fp32 = pr.out_dtype == KVATTN_OUT_FP32;
    a.B = pr.B;
    a.q_len = pr.q_len;
    a.H = pr.H;
    a.NU = pr.NU;
    a.dn = pr.dn;
    a.dr = pr.dr;
    a.row = pr.row;
    a.kv_planes = pr.kv_planes;
    a.HPU = pr.HPU;
    a.HU = pr.HU;
    a.mpps = pr.mpps;
    a.num_pages = pr.num_pages;
    a.max_seq_len = pr.max_seq_len;
    a.num_splits = pl.pub.num_splits;
    a.pages_per_split = pl.pub.pages_per_split;
    a.head_chunks = pl.head_chunks;
    a.latent = pr.latent;
    a.mlra = pr.mlra;
    a.scale_log2 = sm_scale * 1.4426950408889634f;

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    auto mark = [&](int i) {
        return !(events && events[i]) ||
               cudaEventRecord(static_cast<cudaEvent_t>(events[i]), s) == cudaSuccess;
    };
    if (!mark(0))
        return KVATTN_ERR_CUDA;
    cudaError_t le;
    switch (pl.pub.kernel) {
    case KVATTN_KERNEL_GQA: le = launch_gqa(a, s); break;
    case KVATTN_KERNEL_GQA_FP8: le = launch_gqa_fp8(a, p->k_scale, p->v_scale, s); break;
    case KVATTN_KERNEL_MQA_TC: le = launch_mqa_mma(a, s); break;
    case KVATTN_KERNEL_LATENT_TC: le = launch_latent_tc(a, pr, s); break;
    case KVATTN_KERNEL_LATENT_PAIR: le = launch_latent_pair(a, s); break;
    default: le = launch_generic(a, pl.head_chunk, s); break;
    }
    if (le != cudaSuccess)
        return KVATTN_ERR_CUDA;
    if (!mark(1))
        return KVATTN_ERR_CUDA;
    if (pl.fused_merge)
        return mark(2) ? KVATTN_OK : KVATTN_ERR_CUDA;

    CombineArgs c{};
    c.po = a.po;
    c.plse = a.plse;
    c.out = out;
    c.lse = lse;
    c.B = pr.B;
    c.H = pr.H;
    c.NU = pr.NU;
    c.Dv = pr.Dv;
    c.HU = pr.HU;
    c.num_splits = pl.pub.num_splits;
    c.mlra = pr.mlra;
    if (pr.branch_out) {
        // every (head, branch) row merged on its own and written in place:
        // out[b][h][r] is row b * H * R + h * R + r, as the partial rows are
        c.mlra = 0;
        c.H = pr.HU;
    }
    c.out_fp32 = pr.out_dtype == KVATTN_OUT_FP32;
    if (launch_combine(c, s) != cudaSuccess)
        return KVATTN_ERR_CUDA;
    if (!mark(2))
        return KVATTN_ERR_CUDA;
    return KVATTN_OK;
}

extern "C" int kvattn_decode(int32_t variant, const kvattn_params *p, const void *q_nope,
                             const void *q_rope, const void *kv_cache, const int32_t *block_table,
                             const int32_t *seq_lens, float sm_scale, void *out, float *lse,
                             void *workspace, size_t workspace_bytes, void *stream)
{
    return kvattn_decode_timed(variant, p, q_nope, q_rope, kv_cache, block_table, seq_lens,
                               sm_scale, out, lse, workspace, workspace_bytes, stream, nullptr);
}

extern "C" int kvattn_get_device_error(const void *workspace, void *stream, int32_t *code)
{
    if (!workspace || !code)
        return KVATTN_ERR_INVALID_ARG;
    int32_t v = 0;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaMemcpyAsync(&v, workspace, sizeof v, cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return KVATTN_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess)
        return KVATTN_ERR_CUDA;
    *code = v;
    return KVATTN_OK;
}
