/*
 * kvattn.h -- C ABI of the B200 decode-attention library (libkvattn.so).
 *
 * One call computes single-token (decode) attention for a batch of sequences
 * over a compressed or shared KV cache held in HBM:
 *
 *   out[b,h] = sum_j softmax_j( sm_scale * q[b,h] . k_j ) v_j     (j < seq_lens[b])
 *
 * MLA explainer (mlqm.cn/news/371735), section 2.3 gives the formula, section
 * 2.2 the concatenations q = [q^C ; q^R], k = [k^C ; k^R] and that values are
 * the latent part only; the MLRA page (aitntnews.com newId=23265) gives the
 * absorbed decode form (MLA paragraph: W_UK absorbed into the query, decode
 * becomes one 576-wide MQA head), the GQA and MQA bullets, the block
 * decomposition and "moving the sum outside" (per-branch attention, branch
 * outputs summed afterwards); the GLA page (jsbsmhs.com/zixun/902167, "Grouped
 * Latent Attention") gives latent heads that each serve one group of query
 * heads.  The MFA page (jsqmd.com/news/79551, "technical breakthrough") gives
 * a single wide KV head, which decodes as MQA.
 *
 * Variants and what a unit of the cache is:
 *   KVATTN_GQA  num_kv KV heads, query head h uses KV head h / (H / num_kv)
 *   KVATTN_MQA  the same with num_kv = 1 (MFA at decode time: one wide head)
 *   KVATTN_MLA  absorbed MLA: key = [latent (d_nope) ; rope key (d_rope)],
 *               value = latent; num_kv = 1
 *   KVATTN_GLA  num_kv = G latent heads of d_nope each plus one shared rope
 *               key; head h uses latent h / (H / G)
 *   KVATTN_MLRA num_kv = R branches of d_nope each plus one shared rope key;
 *               every head attends every branch with its own query slice and
 *               the R normalised branch outputs are summed (latent space)
 *   KVATTN_GTA  num_kv tied states of d_nope: the cached vector of group g is
 *               both key and value for heads g*H/G .. (GTA/GLA page, "Grouped
 *               Tied Attention"); num_kv = 1 with one wide head is the MFA
 *               page's key reuse (MFA-KR)
 *
 * Memory (all device pointers, row-major, caller-owned):
 *   q_nope     bf16 [B][Q][H][d_nope]        (MLRA [B][Q][H][R][d_nope]), Q = q_len
 *   q_rope     bf16 [B][Q][H][d_rope]        (MLRA [B][Q][H][R][d_rope]); NULL when
 *              d_rope == 0 (GQA/MQA)
 *   kv_cache   latent variants: bf16 [num_pages][page_size][num_kv*d_nope + d_rope],
 *              each token row [c_0 | ... | c_{num_kv-1} | k_rope];
 *              GQA/MQA: bf16 [num_pages][2 (K, V)][page_size][num_kv][d_nope];
 *              GTA: bf16 [num_pages][page_size][num_kv][d_nope] (one tied plane);
 *              GQA with cache_dtype FP8_E4M3: the GQA layout with one e4m3 byte
 *              per element
 *   block_table int32 [B][max_pages_per_seq]: physical page of each logical
 *              64-token page; NULL = contiguous cache, sequence b owns pages
 *              b*max_pages_per_seq .. b*max_pages_per_seq + max_pages_per_seq-1
 *   seq_lens   int32 [B], 0 <= seq_lens[b] <= max_seq_len (read on the device)
 *   out        [B][Q][H][d_nope], bf16 (round to nearest even) or fp32
 *   lse        fp32 [B][Q][H] (MLRA [B][Q][H][R]), natural log of the softmax
 *              denominator including sm_scale; may be NULL
 *   workspace  device scratch of kvattn_workspace_size() bytes, 256-byte
 *              aligned, prepared once with kvattn_workspace_init()
 *
 * Token j of sequence b is slot j % 64 of page block_table[b][j / 64].
 * Slots past seq_lens[b] may hold anything (NaN included) and never reach a
 * result.  An empty sequence yields out = 0 and lse = -inf.
 *
 * Several query tokens per sequence (q_len = Q > 1: speculative or
 * multi-token-prediction decode; the GLA page contrasts query length 1 with
 * longer queries): the Q newest tokens of each sequence are already in the
 * cache (seq_lens counts them), and query position i (0-based) attends the
 * cache up to and including its own token, seq_lens[b] - (Q - 1 - i) tokens
 * (causal).  Each position reads its prefix of the cache on its own.
 *
 * Conventions: every call is asynchronous on `stream` (a cudaStream_t, NULL =
 * legacy default stream) and returns a status before or after enqueueing;
 * nothing is allocated per call and no host synchronisation happens except in
 * kvattn_get_device_error().  Calls on different streams with different
 * workspaces may run concurrently.  Bad arguments return a negative status
 * without launching anything.  Bad data found on the device (a page id outside
 * [0, num_pages), a sequence longer than max_seq_len) sets a bit in the
 * workspace error word; the offending page is skipped, nothing traps.
 */
#ifndef KVATTN_H
#define KVATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum kvattn_variant {
    KVATTN_GQA = 0,
    KVATTN_MQA = 1,
    KVATTN_MLA = 2,
    KVATTN_GLA = 3,
    KVATTN_MLRA = 4,
    KVATTN_GTA = 5
};

enum kvattn_out_dtype { KVATTN_OUT_BF16 = 0, KVATTN_OUT_FP32 = 1 };

/* Element type of the KV cache.  An fp8 cache follows the GTA/GLA page
 * ("Mamba核心作者新作…", the 236B serving test run in FP8) and the MFA page
 * ("突破大模型推理瓶颈…", closing paragraph: quantisation as the next step);
 * neither fixes a format, so the reading here is e4m3 with one scale per
 * tensor.  FP8_E4M3 (GQA with 4 heads per KV head of 128): one byte per
 * element (sign, 4 exponent bits with bias 7, 3 mantissa bits, subnormals at
 * exponent 0; 0x7F / 0xFF are NaN), the key is k_scale * K8, the value
 * v_scale * V8.  The pool layout is the GQA one with byte elements
 * ([num_pages][2][64][num_kv][128] bytes, 16-byte aligned base).  The query
 * stays bf16 and is used as f16 inside the kernel: |q| must stay below 65504. */
enum kvattn_cache_dtype { KVATTN_CACHE_BF16 = 0, KVATTN_CACHE_FP8_E4M3 = 1 };

enum kvattn_status {
    KVATTN_OK = 0,
    KVATTN_ERR_INVALID_ARG = -1,       /* null pointer, bad size, inconsistent shape */
    KVATTN_ERR_UNSUPPORTED = -2,       /* valid request outside what the kernels cover */
    KVATTN_ERR_WORKSPACE_TOO_SMALL = -3,
    KVATTN_ERR_MISALIGNED = -4,        /* a pointer breaks the alignment rules below */
    KVATTN_ERR_CUDA = -5               /* a CUDA launch or copy reported an error */
};

/* Bits of the device error word (kvattn_get_device_error). */
enum kvattn_device_error {
    KVATTN_DEVERR_PAGE_OUT_OF_RANGE = 1, /* block_table entry outside [0, num_pages): page skipped */
    KVATTN_DEVERR_SEQ_TOO_LONG = 2,      /* seq_lens[b] > max_seq_len: clamped to max_seq_len */
    KVATTN_DEVERR_WAIT_TIMEOUT = 4,      /* a bounded wait on an mbarrier ran out: tile skipped */
    KVATTN_DEVERR_POS_OUT_OF_RANGE = 8   /* kvattn_append_kv: a position outside the sequence's
                                            pages: that token skipped */
};

/* Which decode kernel a plan uses. */
enum kvattn_kernel {
    KVATTN_KERNEL_GENERIC = 0,   /* CUDA-core split-KV kernel, any supported shape */
    KVATTN_KERNEL_GQA = 1,       /* GQA kernel: TMA-staged pages, warp-level bf16 MMAs
                                    (m16n8k16), parts merged in the last CTA of each group */
    KVATTN_KERNEL_LATENT_TC = 2, /* tcgen05/TMEM latent kernel, one CTA per group or branch
                                    (GLA, MLRA) */
    KVATTN_KERNEL_MQA_TC = 3,    /* tensor-core MQA kernel (one wide KV head) */
    KVATTN_KERNEL_LATENT_PAIR = 4, /* tcgen05/TMEM MLA kernel (512 + 64) on a 2-CTA cluster:
                                      each CTA scores half of every page and keeps half of
                                      the value columns */
    KVATTN_KERNEL_GQA_FP8 = 5      /* GQA over an fp8 (e4m3) cache: TMA-staged byte tiles widened
                                      to f16 per warp, warp-level f16 MMAs, in-kernel merge */
};

/*
 * Problem description.  Alignment rules: q_nope, q_rope, kv_cache and out
 * 16-byte aligned; lse 4-byte aligned; workspace 256-byte aligned.
 * d_nope and d_rope must be multiples of 8; d_nope <= 512, d_rope <= 128.
 * page_size must be 64.  max_seq_len is a host-side bound on seq_lens used to
 * size the launch (no host read of device memory happens).  num_splits = 0
 * lets the library choose how many parts each context is split into; a
 * positive value forces it (clamped to the pages of the longest sequence).
 */
typedef struct {
    int32_t batch;             /* B >= 1 */
    int32_t num_q_heads;       /* H >= 1 */
    int32_t num_kv;            /* KV heads (GQA/MQA), 1 (MLA), groups G (GLA), branches R (MLRA) */
    int32_t d_nope;            /* head dim (GQA/MQA) or latent width per group/branch */
    int32_t d_rope;            /* width of the shared rope key; 0 for GQA/MQA */
    int32_t page_size;         /* 64 */
    int32_t max_pages_per_seq; /* block_table row stride; capacity = max_pages_per_seq * 64 */
    int32_t num_pages;         /* pages in the pool (bounds check of block_table) */
    int32_t max_seq_len;       /* >= every seq_lens[b]; <= capacity */
    int32_t num_splits;        /* 0 = library choice, > 0 forces */
    int32_t out_dtype;         /* kvattn_out_dtype */
    int32_t q_len;             /* query tokens per sequence, 1..64 (0 means 1); batch * q_len
                                  <= 65535 */
    int32_t branch_out;        /* MLRA only (0 elsewhere): 1 = out holds the R normalised branch
                                  outputs side by side, [B][Q][H][R][d_nope], instead of their
                                  sum, for an up-projection with one W_UV block per branch
                                  (kvattn_head_proj) */
    int32_t cache_dtype;       /* kvattn_cache_dtype; FP8_E4M3 only for GQA with 4 query heads
                                  per KV head of 128 (else UNSUPPORTED) */
    float k_scale;             /* fp8 cache: key = k_scale * stored byte value (> 0, finite) */
    float v_scale;             /* fp8 cache: value = v_scale * stored byte value (> 0, finite);
                                  both ignored for a bf16 cache */
} kvattn_params;

/* What kvattn_decode will launch for a problem (see kvattn_get_plan). */
typedef struct {
    int32_t kernel;            /* kvattn_kernel */
    int32_t num_splits;        /* parts per context */
    int32_t pages_per_split;   /* 64-token pages per part */
    int32_t ctas;              /* CTAs of the decode launch */
    int32_t launches;          /* kernel launches per kvattn_decode call */
    int32_t header_bytes;      /* leading workspace bytes that must be zero before a call
                                  (error word and part counters); calls leave them zero */
    uint64_t workspace_bytes;  /* required workspace */
} kvattn_plan;

/* Fill *plan for (variant, p).  Returns KVATTN_OK or INVALID_ARG/UNSUPPORTED.
 * Host only: no device memory is touched and nothing is enqueued.  The plan is
 * sized for the current device's SM count, queried once per device through
 * the CUDA runtime (148, a B200, when no device can be queried). */
int kvattn_get_plan(int32_t variant, const kvattn_params *p, kvattn_plan *plan);

/* Bytes of workspace kvattn_decode needs for (variant, p): a 256-byte header
 * holding the device error word, one counter per (sequence, KV head / unit)
 * for kernels that merge their own parts, then the per-part lse
 * [B][splits][rows] and normalised outputs [B][splits][rows][d_nope] in fp32
 * (rows = H, or H*R for MLRA).  Host only. */
int kvattn_workspace_size(int32_t variant, const kvattn_params *p, size_t *bytes);

/* Zero the whole workspace on `stream`.  Call once after allocating a
 * workspace, and again after a device error (a call cut short may leave its
 * part counters non-zero). */
int kvattn_workspace_init(void *workspace, size_t workspace_bytes, void *stream);

/*
 * Decode attention, enqueued on `stream`: a split-KV pass that writes one
 * normalised partial output and lse per (sequence, head[, branch], part)
 * into the workspace, and a merge of the parts by their lse
 * (flash-decoding) that sums the MLRA branches, places GLA group heads and
 * casts to out_dtype.  The GQA kernel merges in the last CTA of each
 * (sequence, KV head) to finish (one launch); the others run a combine pass
 * (two launches; kvattn_get_plan reports which).  The combine pass is a
 * programmatic dependent launch of the split pass: the GPU may schedule it
 * while the split pass drains, and it waits on the device until that pass
 * has completed and its writes are visible.  Returns KVATTN_OK once
 * enqueued, a negative status (nothing enqueued) for bad arguments,
 * KVATTN_ERR_CUDA if a launch failed.
 */
int kvattn_decode(int32_t variant, const kvattn_params *p, const void *q_nope, const void *q_rope,
                  const void *kv_cache, const int32_t *block_table, const int32_t *seq_lens,
                  float sm_scale, void *out, float *lse, void *workspace, size_t workspace_bytes,
                  void *stream);

/* kvattn_decode that also records caller-created cudaEvent_t handles on
 * `stream`: events[0] before the split pass, events[1] after it (for the
 * kernels that merge their own parts this includes the merge), events[2]
 * after the combine pass, or right after events[1] when there is none (a
 * NULL entry is skipped; events may be NULL).  Used to time each pass on the launching
 * stream; an event recorded between the passes makes them run strictly one
 * after the other.  Same arguments, statuses and results as kvattn_decode. */
int kvattn_decode_timed(int32_t variant, const kvattn_params *p, const void *q_nope,
                        const void *q_rope, const void *kv_cache, const int32_t *block_table,
                        const int32_t *seq_lens, float sm_scale, void *out, float *lse,
                        void *workspace, size_t workspace_bytes, void *stream,
                        void *const *events);

/*
 * Size of the device scratch array behind kvattn_decode_noalloc (32 MiB).
 */
#define KVATTN_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)

/*
 * kvattn_decode_noalloc -- the same decode attention for callers that cannot
 * allocate device memory.  The pages describe no such interface; it has no
 * counterpart there.
 *
 * Who needs it: callers that cannot hand the library a workspace, because
 * they may not call cudaMalloc at all -- a serving engine that has already
 * reserved all of HBM for its own cache pool, a plugin host that gives a
 * library only its input and output buffers, or a latency-critical path where
 * an allocation (which can synchronise the device) is not acceptable.
 *
 * The caller passes the inputs and outputs exactly as for kvattn_decode
 * (same layouts, alignment and statuses) but no workspace.  The scratch lives
 * in one device array of KVATTN_NOALLOC_SCRATCH_BYTES inside the library,
 * which every GPU that loads the library holds until the process exits.
 * Nothing is allocated by this call.  A problem whose workspace does not fit
 * is run with fewer parts per context when num_splits is 0; if it still does
 * not fit, or a forced num_splits does not fit, the call returns
 * KVATTN_ERR_WORKSPACE_TOO_SMALL and enqueues nothing.
 *
 * The first call on a device (that device current) looks up the array's
 * device address; make that first call before any stream capture.  Under lazy
 * module loading (the CUDA default) that first call is also when the array is
 * reserved on the device, so make it before the caller claims the rest of
 * HBM.  The address is kept per device and is stale after cudaDeviceReset.
 * All calls share the one array, which keeps the last call's contents: calls
 * ordered on one stream are safe, calls that overlap on the GPU race on it.
 * Arguments are checked as kvattn_decode checks them before anything is
 * enqueued: a refused call (any negative status) leaves the array untouched.
 * Each call clears the device error word at its start; device_error (device
 * memory, 4 bytes, may be NULL) receives that call's kvattn_device_error bits.
 */
int kvattn_decode_noalloc(int32_t variant, const kvattn_params *p, const void *q_nope,
                          const void *q_rope, const void *kv_cache, const int32_t *block_table,
                          const int32_t *seq_lens, float sm_scale, void *out, float *lse,
                          int32_t *device_error, void *stream);

/*
 * kvattn_selftest_bounded_wait -- check, on the device, the bounded mbarrier
 * wait every decode kernel uses.  No page defines it: it tests the library's
 * own failure detection (a wait that runs out sets
 * KVATTN_DEVERR_WAIT_TIMEOUT and returns instead of hanging the GPU).
 *
 * Enqueues on `stream` one single-warp kernel that initialises two mbarriers,
 * completes the phase of one of them and then waits, each wait capped at
 * `tries` attempts (1 <= tries <= 65536): first on the completed phase, which
 * must succeed, then on the other barrier, which no thread ever arrives on and
 * must run out.  It ORs into *result (device memory, 4 bytes, caller-zeroed):
 * KVATTN_DEVERR_WAIT_TIMEOUT when the second wait gave up as it should, and
 * KVATTN_SELFTEST_MISSED_PHASE when the first wait failed to see a completed
 * phase.  A correct library leaves exactly KVATTN_DEVERR_WAIT_TIMEOUT.
 * Returns INVALID_ARG / MISALIGNED for bad arguments (nothing enqueued) and
 * KVATTN_ERR_CUDA if the launch failed.
 */
#define KVATTN_SELFTEST_MISSED_PHASE 256
int kvattn_selftest_bounded_wait(int32_t *result, int32_t tries, void *stream);

/*
 * The steps either side of attention.
 *
 * kvattn_rope: rotary position embedding in place (MLA explainer section 2.2:
 * the position branch's q^R and k^R are rotated; the pages print no formula,
 * and this is the embedding's original form).  x is bf16 [rows][row_elems];
 * in each row the slice [rot_offset, rot_offset + rot_dim) is taken as
 * pairs (x[2i], x[2i+1]) and pair i is turned by the angle
 * pos * rope_base^(-2i/rot_dim), pos = pos[row / rows_per_pos] (int32, any
 * value; used as given).  Angle and turn in double precision, one rounding
 * to bf16 (nearest even).  For the absorbed query of MLA/GLA (q_rope
 * [B][Q][H][d_rope]): rows = B*Q*H, row_elems = rot_dim = d_rope,
 * rows_per_pos = H, pos[B*Q] the query tokens' positions; MLRA rows carry R
 * slices each (rows = B*Q*H*R, rows_per_pos = H*R).  rot_offset, rot_dim and
 * row_elems even, rope_base > 1, x and pos 4-byte aligned; rows = 0 does
 * nothing.  INVALID_ARG / MISALIGNED before anything is enqueued.
 */
int kvattn_rope(void *x, int32_t rows, int32_t row_elems, int32_t rot_offset, int32_t rot_dim,
                int32_t rows_per_pos, const int32_t *pos, float rope_base, void *stream);

/*
 * kvattn_append_kv: write the newest tokens of each sequence into the paged
 * cache decode reads (MLA explainer section 2.4: the compact latent is what
 * the cache keeps).  p gives the cache geometry (batch, q_len = tokens per
 * sequence, num_kv, d_nope, d_rope, max_pages_per_seq, num_pages; the other
 * fields are checked as for decode).  new_kv, bf16, caller-owned:
 *   latent variants  [B][Q][num_kv*d_nope + d_rope], [c_0 | ... | k^R] with
 *                    k^R not yet rotated;
 *   GQA/MQA          [B][Q][2][num_kv][d_nope], K then V;
 *   GTA              [B][Q][num_kv][d_nope], the tied vectors (stored as
 *                    given: rope_base must be 0).
 * pos int32 [B][Q]: the cache position of each token (slot pos % 64 of page
 * block_table[b][pos / 64]; block_table NULL = contiguous, as in decode).
 * rope_base > 1 rotates k^R (latent) or every K head (GQA/MQA) at its
 * position on the way in, exactly as kvattn_rope does; rope_base = 0 stores
 * the rows as given.  Latent parts and V are copied bit for bit.  A position
 * outside [0, max_pages_per_seq * 64) sets KVATTN_DEVERR_POS_OUT_OF_RANGE, a
 * page id outside [0, num_pages) KVATTN_DEVERR_PAGE_OUT_OF_RANGE, in
 * *device_error (int32 device word, may be NULL), and that token is skipped.
 * new_kv and kv_cache 16-byte aligned.  Seq_lens are not touched: the caller
 * counts the new tokens in before the next decode.
 */
int kvattn_append_kv(int32_t variant, const kvattn_params *p, const void *new_kv, const int32_t *pos,
                     const int32_t *block_table, void *kv_cache, float rope_base, int32_t *device_error,
                     void *stream);

/*
 * kvattn_head_proj: y[r][h][:] = x[r][h][:] @ w[h] for every row r and head h,
 * bf16 inputs, fp32 accumulation on the tensor cores, y bf16 (nearest even)
 * or fp32 (out_dtype).  x [rows][heads][k], w [heads][k][n], y
 * [rows][heads][n], row-major, 16-byte aligned; k and n multiples of 64.
 *   Query absorption (MLRA page, MLA paragraph: W_UK folded into the query):
 *     x = q^C [B*Q][H][d_h], w = W_UK [H][d_h][d_c] (per MLRA head the R
 *     branch blocks side by side, n = R*d_c), y = q_nope for decode.
 *   Up-projection (MLA explainer section 2.3: outputs weight c W_UV):
 *     x = decode's out [B*Q][H][d_c] (MLRA with branch_out: [B*Q][H][R*d_c]),
 *     w = W_UV [H][d_c][d_v] (MLRA: the R branch blocks stacked, k = R*d_c,
 *     so the branch sum of "moving the sum outside" is part of the
 *     contraction), y the attention output per head.
 * A wait that runs out sets KVATTN_DEVERR_WAIT_TIMEOUT in *device_error (may
 * be NULL).  rows = 0 does nothing.
 */
int kvattn_head_proj(const void *x, const void *w, void *y, int32_t out_dtype, int32_t rows, int32_t heads,
                     int32_t k, int32_t n, int32_t *device_error, void *stream);

/* Copy the device error word to *code (0 = none, else kvattn_device_error
 * bits).  Synchronises `stream`.  Returns KVATTN_ERR_CUDA if the copy
 * failed. */
int kvattn_get_device_error(const void *workspace, void *stream, int32_t *code);

/* Static, human-readable name of a status code. */
const char *kvattn_status_string(int status);

/* Library ABI version (major * 100 + minor): 202 (kvattn_params carries q_len,
 * branch_out and the cache element type with its scales; the steps either side:
 * kvattn_rope, kvattn_append_kv, kvattn_head_proj). */
int kvattn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KVATTN_H */
