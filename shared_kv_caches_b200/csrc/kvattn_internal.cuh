// Internal declarations shared by the decode, combine and host sources of
// libkvattn.so.  Nothing here is part of the C ABI (see include/kvattn.h).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kvattn.h"

namespace kvattn {

constexpr int kPage = 64;               // tokens per cache page
constexpr int kNumSMs = 148;            // B200 streaming multiprocessors
constexpr size_t kWsHeader = 256;       // workspace header: device error word
constexpr int kMaxSplits = 1024;

// Validated problem, host side.
struct Problem {
    int variant;
    int B, H, NU, dn, dr;
    int Dk, Dv;        // key width (d_nope + d_rope) and value width (d_nope)
    int row;           // elements per token row of a page (per K or V plane for GQA/MQA)
    int HPU;           // query heads served by one unit (KV head / group / branch)
    int HU;            // partial rows per sequence: H, or H*R for MLRA
    int mpps, num_pages, max_seq_len, out_dtype;
    bool latent, mlra, paged;
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
    int B, H, NU, dn, dr, row, HPU, HU;
    int mpps, num_pages, max_seq_len;
    int num_splits, pages_per_split, head_chunks;
    int latent, mlra;
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

// Launchers (each returns the launch's cudaError_t).
cudaError_t launch_generic(const DecodeArgs &a, int head_chunk, cudaStream_t st);
size_t generic_smem_bytes(const Problem &pr, int head_chunk);
cudaError_t launch_combine(const CombineArgs &a, cudaStream_t st);
bool gqa_supported(const Problem &pr);
cudaError_t launch_gqa(const DecodeArgs &a, cudaStream_t st);
bool mqa_mma_supported(const Problem &pr);
cudaError_t launch_mqa_mma(const DecodeArgs &a, cudaStream_t st);
int latent_tc_slots(const Problem &pr);
int latent_tc_page_multiple(const Problem &pr);
int latent_tc_max_pages_per_split();
cudaError_t launch_latent_tc(const DecodeArgs &a, const Problem &pr, cudaStream_t st);

}  // namespace kvattn
