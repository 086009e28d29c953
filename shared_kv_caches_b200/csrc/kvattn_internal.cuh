// Internal declarations shared by the decode, combine and host sources of
// libkvattn.so.  Nothing here is part of the C ABI (see include/kvattn.h).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "kvattn.h"

namespace kvattn {

constexpr int kPage = 64;               // tokens per cache page
constexpr int kDefaultSMs = 148;        // B200; used when no device can be queried
constexpr size_t kWsHeader = 256;       // workspace header: device error word
constexpr int kMaxSplits = 1024;
constexpr int kMaxQueryLen = 64;        // query tokens per sequence in one call

// Validated problem, host side.
struct Problem {
    int variant;
    int B, H, NU, dn, dr;  // B: rows = sequences x query tokens
    int q_len;         // query tokens per sequence
    int Dk, Dv;        // key width (d_nope + d_rope) and value width (d_nope)
    int row;           // elements per token row of a page (per K or V plane for GQA/MQA)
    int HPU;           // query heads served by one unit (KV head / group / branch)
    int HU;            // partial rows per sequence: H, or H*R for MLRA
    int mpps, num_pages, max_seq_len, out_dtype;
    bool latent, mlra, paged;
    bool branch_out;   // MLRA: the R branch outputs side by side instead of their sum
    int kv_planes;     // GQA/MQA pages: 2 (K, V); GTA: 1 (the tied vector is key and value)
};

// Arguments of every decode kernel.  Partial results go to the workspace as
// plse[b][split][hu] and po[b][split][hu][Dv] (fp32, normalised).
struct DecodeArgs {
    const __nv_bfloat16 *q_nope;
    const __nv_bfloat16 *q_rope;
    const __nv_bfloat16 *kv;
    const int32_t *block_table;   // nullptr: contiguous cache
    const int32_t *seq_lens;
    float *po;
    float *plse;
    int *err;
    int *tickets;                 // per (sequence, unit): parts finished (in-kernel merge)
    void *out;                    // final output and lse, for kernels that merge their own parts
    float *lse_out;
    int out_fp32;
    int B, H, NU, dn, dr, row, HPU, HU;
    int mpps, num_pages, max_seq_len;
    int num_splits, pages_per_split, head_chunks;
    int latent, mlra;
    int q_len;                    // query tokens per sequence; B counts (sequence, position) rows
    int kv_planes;                // GQA/MQA pages: 2 (K, V); GTA: 1 (keys are the values)
    float scale_log2;             // sm_scale * log2(e): scores kept in base 2
};

struct CombineArgs {
    const float *po;
    const float *plse;
    void *out;
    float *lse;
    int B, H, NU, Dv, HU, num_splits, mlra, out_fp32;
};

__device__ __forceinline__ void raise_error(int *err, int bit) { atomicOr(err, bit); }

// Row v of a decode call is query position v % q_len of sequence v / q_len.
// Position i of the q_len newest tokens attends the cache up to and
// including itself: seq_lens[s] - (q_len - 1 - i) tokens (causal).  A
// sequence longer than max_seq_len sets the error bit (in the first CTA of
// its rows that reads it) and is clamped.
__device__ __forceinline__ int row_context(const DecodeArgs &a, int v, bool report)
{
    const int s = v / a.q_len, pos = v % a.q_len;
    int L = a.seq_lens[s];
    if (L > a.max_seq_len) {
        if (report)
            raise_error(a.err, KVATTN_DEVERR_SEQ_TOO_LONG);
        L = a.max_seq_len;
    }
    return max(L - (a.q_len - 1 - pos), 0);
}

// Physical page of logical page pi of row v's sequence.
__device__ __forceinline__ long long row_page(const DecodeArgs &a, int v, int pi)
{
    const long long s = v / a.q_len;
    return a.block_table ? (long long)a.block_table[s * a.mpps + pi] : s * a.mpps + pi;
}

// Programmatic dependent launch: a decode kernel lets the combine pass queued
// behind it be scheduled at once (its blocks then wait in pdl_wait_primary
// until every decode CTA has finished and its writes are visible), so the
// combine's launch overlaps the decode's tail.
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait_primary() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Merge of the parts of one (sequence b, rows hu0 .. hu0 + nrows - 1) group,
// run by the last CTA of the group to finish: lse = ln sum_s exp(lse_s),
// out = sum_s exp(lse_s - lse) o_s, cast to the output type.  w is shared
// scratch of nrows * num_splits floats; tid / nthr index the threads taking
// part, which meet at named barrier bar_id.  Partial rows written by other
// CTAs are read past L1.
__device__ __forceinline__ void merge_group(const DecodeArgs &a, int b, int hu0, int nrows, int Dv, float *w, int tid,
                                            int nthr, int bar_id)
{
    const int S = a.num_splits;
    const int warp = tid >> 5, lane = tid & 31, nwarps = nthr >> 5;
    for (int r = warp; r < nrows; r += nwarps) {
        const float *pl = a.plse + (size_t)b * S * a.HU + hu0 + r;
        float mx = -INFINITY;
        for (int s = lane; s < S; s += 32)
            mx = fmaxf(mx, __ldcg(pl + (size_t)s * a.HU));
        for (int o = 16; o; o >>= 1)
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        float sum = 0.f;
        for (int s = lane; s < S; s += 32) {
            const float e = mx == -INFINITY ? 0.f : expf(__ldcg(pl + (size_t)s * a.HU) - mx);
            w[r * S + s] = e;
            sum += e;
        }
        for (int o = 16; o; o >>= 1)
            sum += __shfl_xor_sync(0xffffffffu, sum, o);
        const float inv = sum > 0.f ? 1.f / sum : 0.f;
        for (int s = lane; s < S; s += 32)
            w[r * S + s] *= inv;
        if (lane == 0 && a.lse_out)
            a.lse_out[(size_t)b * a.HU + hu0 + r] = (mx == -INFINITY || !(sum > 0.f)) ? -INFINITY : mx + logf(sum);
    }
    asm volatile("bar.sync %0, %1;" ::"r"(bar_id), "r"(nthr) : "memory");
    for (int idx = 4 * tid; idx < nrows * Dv; idx += 4 * nthr) {
        const int r = idx / Dv, d = idx % Dv;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int s = 0; s < S; ++s) {
            const float ws = w[r * S + s];
            const float4 v = __ldcg(reinterpret_cast<const float4 *>(
                a.po + (((size_t)b * S + s) * a.HU + hu0 + r) * Dv + d));
            acc.x = fmaf(ws, v.x, acc.x);
            acc.y = fmaf(ws, v.y, acc.y);
            acc.z = fmaf(ws, v.z, acc.z);
            acc.w = fmaf(ws, v.w, acc.w);
        }
        const size_t o = ((size_t)b * a.H + hu0 + r) * Dv + d;
        if (a.out_fp32) {
            *reinterpret_cast<float4 *>(static_cast<float *>(a.out) + o) = acc;
        } else {
            const __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y);
            const __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z, acc.w);
            uint2 packed;
            packed.x = *reinterpret_cast<const uint32_t *>(&lo);
            packed.y = *reinterpret_cast<const uint32_t *>(&hi);
            *reinterpret_cast<uint2 *>(static_cast<__nv_bfloat16 *>(a.out) + o) = packed;
        }
    }
}

// Count this CTA's part of group `ticket_idx` as finished (after its partial
// writes); true in the one CTA that finished last, which then owns the merge
// and resets the counter for the next call.  All nthr threads call it.
__device__ __forceinline__ bool finish_part(const DecodeArgs &a, int ticket_idx, int *flag, int tid, int nthr,
                                            int bar_id)
{
    __threadfence();
    asm volatile("bar.sync %0, %1;" ::"r"(bar_id), "r"(nthr) : "memory");
    if (tid == 0) {
        const int t = atomicAdd(&a.tickets[ticket_idx], 1);
        *flag = t == a.num_splits - 1;
    }
    asm volatile("bar.sync %0, %1;" ::"r"(bar_id), "r"(nthr) : "memory");
    const bool last = *flag != 0;
    if (last) {
        __threadfence();
        if (tid == 0)
            a.tickets[ticket_idx] = 0;
    }
    return last;
}

// Streaming multiprocessors of the current device (queried once per device
// through the runtime; kDefaultSMs when there is no device).
int sm_count();

// Argument checks shared by every decode entry point: the problem, the
// pointers and their alignment, sm_scale.  Returns a kvattn_status; nothing
// is enqueued.
// Shape checks of kvattn_params (the Problem every entry point works from).
int validate_params(int32_t variant, const kvattn_params *p, Problem *pr);
int validate_call(int32_t variant, const kvattn_params *p, const void *q_nope, const void *q_rope,
                  const void *kv_cache, const int32_t *block_table, const int32_t *seq_lens,
                  float sm_scale, const void *out, const float *lse, const void *workspace,
                  Problem *pr);

// Launchers (each returns the launch's cudaError_t).
cudaError_t launch_generic(const DecodeArgs &a, int head_chunk, cudaStream_t st);
size_t generic_smem_bytes(const Problem &pr, int head_chunk);
cudaError_t launch_combine(const CombineArgs &a, cudaStream_t st);
bool gqa_supported(const Problem &pr);
cudaError_t launch_gqa(const DecodeArgs &a, cudaStream_t st);
bool mqa_mma_supported(const Problem &pr);
cudaError_t launch_mqa_mma(const DecodeArgs &a, cudaStream_t st);
bool latent_pair_supported(const Problem &pr);
cudaError_t launch_latent_pair(const DecodeArgs &a, cudaStream_t st);
int latent_tc_slots(const Problem &pr);
int latent_tc_page_multiple(const Problem &pr);
int latent_tc_max_pages_per_split();
cudaError_t launch_latent_tc(const DecodeArgs &a, const Problem &pr, cudaStream_t st);

}  // namespace kvattn
