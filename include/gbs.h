/*
 * gbs.h — C ABI of the gated block-sparse causal attention library (libgbs.so).
 *
 * The operation (SAS, "Simple Attention Sparsification via End-to-End
 * Optimization of Context Ranking"):
 *   - selector scores S over earlier key blocks become normalised softmax gates
 *     g, applied in log form inside the attention softmax (NeurIPS 2026 poster
 *     page, Abstract; Hugging Face paper page, Abstract);
 *   - logit z_ij = scale * q_i.k_j + log g[r(i), c(j)] for keys in an attended
 *     historical block c < r, + 0 for keys of the always-retained current block
 *     r with j <= i, and -inf otherwise (ai.viyan.live, "SAS Learns Token
 *     Importance for Sparse Attention", section "The Logit Injection Mechanism");
 *   - training mode attends every historical block and the backward pass
 *     returns dQ, dK, dV and dS, the gradient through the gate softmax into the
 *     scores (same blog page and section; poster Abstract: all context units
 *     active during training);
 *   - sparse mode attends only the Top-K historical blocks by score plus the
 *     current block (poster Abstract: fixed attention budget; HF page Abstract:
 *     hard Top-K). Gates are renormalised over the selected blocks.
 *   - threshold mode is the dynamic variant (blog section "Implementation and
 *     Efficiency": only blocks whose importance passes a threshold are
 *     computed): a query block keeps the historical blocks whose training-mode
 *     gate exp(S[r,c]) / sum_{c'<r} exp(S[r,c']) is at least tau, at most
 *     topk of them (largest scores first), i.e. Top-k with
 *     k = min(topk, #{c < r : gate >= tau}); gates are then renormalised over
 *     the kept blocks as in sparse mode. The comparison is taken in fp32 as
 *     S[r,c] - lse_r >= ln(tau), lse_r the fp32 row log-sum-exp.
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers (cudaMalloc / torch memory),
 *     contiguous row-major in the layouts given per function, 16-byte aligned.
 *     The caller owns every buffer, including the workspace `ws`; the library
 *     never allocates, frees or synchronises (gbs_check excepted).
 *   - `stream` is a cudaStream_t (NULL = legacy default stream). Work is
 *     enqueued asynchronously.
 *   - Arguments are validated before any launch; on failure the function
 *     returns a status and leaves every output untouched; gbs_last_error()
 *     then describes the failing argument.
 *   - Launch failures return GBS_ERR_CUDA. Errors detected on the device
 *     (a bounded wait that expired) are recorded in the workspace's error word
 *     and reported by gbs_check().
 *   - Layouts: Q, O, dO, dQ [B, Hq, N, d]; K, V, dK, dV [B, Hkv, N, d];
 *     LSE [B, Hq, N] fp32; S, dS [B, Hq, Nb, Nb] fp32 with Nb = N / block
 *     (only entries with c < r are read; dS is written 0 elsewhere).
 *     q-head h reads kv-head h / (Hq / Hkv).
 *   - Supported: d in {64, 128}; block == 64; N % 64 == 0 (training/prefill);
 *     Hq % Hkv == 0; 0 <= topk <= GBS_MAX_TOPK; dtype bf16 (tensor-core path)
 *     or fp32 (exact SIMT path). S must be finite. B * Hq * N < 2^31 (token
 *     rows are 32-bit TMA coordinates); larger problems return
 *     GBS_ERR_INVALID_ARG.
 */
#ifndef GBS_H_
#define GBS_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define GBS_API __attribute__((visibility("default")))
#else
#define GBS_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

#define GBS_VERSION_MAJOR 0
#define GBS_VERSION_MINOR 1
#define GBS_MAX_TOPK 256

typedef enum gbs_status {
  GBS_OK = 0,
  GBS_ERR_INVALID_ARG = 1,   /* a shape, pointer, alignment or size is invalid  */
  GBS_ERR_UNSUPPORTED = 2,   /* valid, but not a configuration this build runs  */
  GBS_ERR_CUDA = 3,          /* a CUDA runtime call or kernel launch failed     */
  GBS_ERR_TIMEOUT = 4,       /* a device-side bounded wait expired (gbs_check)  */
  GBS_ERR_WORKSPACE = 5,     /* workspace missing or smaller than required      */
  GBS_ERR_DEVICE_CHECK = 6   /* debug build only: a device-side index check
                                failed (the access was clamped; gbs_check)    */
} gbs_status;

typedef enum gbs_mode { GBS_TRAIN = 0, GBS_SPARSE = 1, GBS_THRESHOLD = 2 } gbs_mode;
typedef enum gbs_dtype { GBS_BF16 = 0, GBS_F32 = 1 } gbs_dtype;
typedef enum gbs_op { GBS_OP_FWD = 0, GBS_OP_BWD = 1, GBS_OP_DECODE = 2 } gbs_op;

typedef struct gbs_params {
  int B;        /* batch                                                     */
  int Hq;       /* query heads                                               */
  int Hkv;      /* key/value heads, Hq % Hkv == 0                            */
  int N;        /* tokens (training / prefill) or cache length L (decode)   */
  int d;        /* head dimension                                            */
  int block;    /* context-unit block size (tokens per block)               */
  int topk;     /* budget K of historical blocks (sparse, threshold, decode) */
  int mode;     /* gbs_mode                                                  */
  int dtype;    /* gbs_dtype of Q, K, V, O, dO, dQ, dK, dV                   */
  float scale;  /* logit scale; 0 selects 1/sqrt(d)                          */
  float tau;    /* threshold mode: gate threshold, 0 < tau <= 1; else unused */
} gbs_params;

/* Version as (major << 16) | minor. */
GBS_API int gbs_version(void);

/* Text of a status code; never NULL. */
GBS_API const char* gbs_status_string(gbs_status s);

/* Description of the last validation failure on the calling thread ("" if none). */
GBS_API const char* gbs_last_error(void);

/* Bytes of workspace `ws` that gbs_fwd / gbs_bwd / gbs_decode need for `op`
 * with these parameters (0 if the parameters are invalid). The workspace must
 * be device memory, 256-byte aligned, and must not be shared by calls that run
 * concurrently. Its first word is the device error word read by gbs_check. */
GBS_API size_t gbs_workspace_bytes(const gbs_params* p, int op);

/* Clears the device error word of `ws` (asynchronous, on `stream`). */
GBS_API gbs_status gbs_clear_error(void* ws, void* stream);

/* Reads the device error word of `ws`: synchronises `stream`, returns GBS_OK
 * or the recorded status (GBS_ERR_TIMEOUT when a bounded wait expired). */
GBS_API gbs_status gbs_check(const void* ws, void* stream);

/* Gate normalisation and Top-K (or threshold) block selection (K1).
 * Normalised softmax gates in log form over the attended historical set
 * (HF page Abstract; blog section "Differentiable Budget Constraints").
 *   S     [B, Hq, Nb, Nb] fp32, row r scores key blocks c < r.
 *   slse  [B, Hq, Nb] fp32 out: ln sum_{c<r} exp S[r, c] (-inf for r = 0);
 *         may be NULL in sparse and threshold modes.
 *   Sparse and threshold modes only (may be NULL in training mode); in
 *   threshold mode read min(topk, r) below as k of the mode's definition:
 *   idx   [B, Hq, Nb, topk] int32 out: A_r ascending, -1 padded. A_r holds the
 *         min(topk, r) blocks c < r with the largest S[r, c]; ties go to the
 *         lower index; -0.0 equals +0.0.
 *   cnt   [B, Hq, Nb] int32 out: |A_r|.
 *   logg  [B, Hq, Nb, topk] fp32 out: S[r, c] - ln sum_{c' in A_r} exp S[r, c'],
 *         0 in the padding. */
GBS_API gbs_status gbs_select(const gbs_params* p, const float* S, int32_t* idx, int32_t* cnt,
                      float* logg, float* slse, void* stream);

/* Gated attention forward (select + attention): softmax attention whose
 * logits carry the log gates of the attended historical blocks and 0 for the
 * current block (blog section "The Logit Injection Mechanism"; poster and HF
 * page Abstracts for the training and Top-K modes; blog section
 * "Implementation and Efficiency" for the threshold mode and the blockwise
 * processing that never forms the N x N matrix).
 *   Q [B,Hq,N,d], K/V [B,Hkv,N,d] in p->dtype; S [B,Hq,Nb,Nb] fp32.
 *   O [B,Hq,N,d] out (p->dtype); LSE [B,Hq,N] fp32 out, natural log of
 *   sum_j exp z_ij with z including scale and bias.
 *   p->mode selects training (every block c < r, gates over all of them),
 *   sparse (Top-K blocks, gates renormalised over them) or threshold (blocks
 *   whose gate reaches p->tau, at most Top-K, gates renormalised).
 *   ws: gbs_workspace_bytes(p, GBS_OP_FWD) bytes. */
GBS_API gbs_status gbs_fwd(const gbs_params* p, const void* Q, const void* K, const void* V,
                   const float* S, void* O, float* LSE, void* ws, size_t ws_bytes,
                   void* stream);

/* Gated attention backward (blog section "The Logit Injection Mechanism": the
 * gradient reaches the scores through the gates inside the softmax).
 *   O, LSE: outputs of gbs_fwd for the same inputs and p. dO [B,Hq,N,d]
 *   (p->dtype). dQ [B,Hq,N,d], dK/dV [B,Hkv,N,d] out (p->dtype; fp32
 *   accumulation). dS [B,Hq,Nb,Nb] fp32 out: dS[r,c'] = G[r,c'] - g[r,c']
 *   sum_{c in A_r} G[r,c] for c' in A_r and 0 elsewhere, where G[r,c] sums
 *   dL/dz over the (r,c) tile and A_r is the attended historical set (all of
 *   c < r in training mode). In sparse and threshold modes (an extension: the
 *   pages train with every block active) A_r is recomputed from S exactly as
 *   gbs_fwd selects it, g is renormalised over A_r, and the selection itself
 *   passes no gradient.
 *   ws: gbs_workspace_bytes(p, GBS_OP_BWD) bytes. */
GBS_API gbs_status gbs_bwd(const gbs_params* p, const void* Q, const void* K, const void* V,
                   const float* S, const void* O, const float* LSE, const void* dO,
                   void* dQ, void* dK, void* dV, float* dS, void* ws, size_t ws_bytes,
                   void* stream);

/* Sparse decode: one query per sequence at position L-1 (L = p->N), the
 * inference-time use of the method with a fixed budget of context blocks per
 * query (poster Abstract) and the current block always retained (HF page
 * Abstract).
 *   q [B,Hq,d]; Kc/Vc [B,Hkv,L,d] (p->dtype); S [B,Hq,Nb] fp32 with
 *   Nb = ceil(L / block): scores of the current block's row over key blocks
 *   c < cur = (L-1)/block. Attends the Top-K (p->topk) historical blocks with
 *   renormalised log gates plus the current block up to L-1 with bias 0.
 *   p->mode GBS_THRESHOLD keeps only those of them whose gate reaches p->tau
 *   (as in gbs_fwd); any other mode value selects plain Top-K.
 *   O [B,Hq,d] out (p->dtype); LSE [B,Hq] fp32 out.
 *   num_splits: partitions of the selected blocks per (b, h); 0 = automatic
 *               (at most 17 blocks per partition, and at least two waves of
 *               resident CTAs).
 *   ws: gbs_workspace_bytes(p, GBS_OP_DECODE) bytes. */
GBS_API gbs_status gbs_decode(const gbs_params* p, const void* q, const void* Kc, const void* Vc,
                      const float* S, void* O, float* LSE, int num_splits, void* ws,
                      size_t ws_bytes, void* stream);

/* Where gbs_decode_ex finds the KV cache and how the q-heads select (a
 * serving-side layout of the decode above; the pages describe long-context
 * inference but no cache layout, so this one is the library's own).
 *   block_table  NULL: Kc/Vc are contiguous [B, Hkv, L, d] as in gbs_decode.
 *                Else a DEVICE array [B, max_blocks] of int32: block c of
 *                sequence b lives in page block_table[b * max_blocks + c], and
 *                Kc/Vc are page pools [num_pages, Hkv, block, d] (one context
 *                block of every kv head per page). Only the first
 *                ceil(L_b / block) entries of a row are read.
 *   max_blocks   row stride of block_table, >= ceil(p->N / block).
 *   num_pages    pages in each pool, with num_pages * Hkv * block < 2^31;
 *                an entry outside [0, num_pages) is
 *                skipped on the device and reported by gbs_check as
 *                GBS_ERR_INVALID_ARG (that sequence's output is then wrong).
 *   seq_lens     NULL: every sequence has length L = p->N. Else a DEVICE array
 *                [B] of int32 lengths L_b in [1, p->N] (p->N is the maximum);
 *                the query of sequence b sits at L_b - 1 and S row entries
 *                c < (L_b - 1) / block are read. A length outside the range
 *                is clamped and reported like a bad page.
 *   group_shared 0: S is [B, Hq, Nb], one selection per q-head (gbs_decode).
 *                1: S is [B, Hkv, Nb], one selection per kv group, used by its
 *                Hq / Hkv q-heads, so each selected key/value block is read
 *                once for the whole group.
 * All fields are read at call time; the arrays must stay valid until the
 * call's work on `stream` has finished. */
typedef struct gbs_kv_layout {
  const int32_t* block_table;
  int max_blocks;
  int num_pages;
  const int32_t* seq_lens;
  int group_shared;
} gbs_kv_layout;

/* gbs_decode over the cache layout `kv` (NULL = gbs_decode). Same workspace
 * size (gbs_workspace_bytes(p, GBS_OP_DECODE)) and outputs as gbs_decode. */
GBS_API gbs_status gbs_decode_ex(const gbs_params* p, const gbs_kv_layout* kv, const void* q,
                                 const void* Kc, const void* Vc, const float* S, void* O,
                                 float* LSE, int num_splits, void* ws, size_t ws_bytes,
                                 void* stream);

/* Profiling hook: while `start`/`stop` (cudaEvent_t, caller-owned) are set for
 * `op`, every call of that op records `start` on its stream immediately before
 * its main attention kernel and `stop` immediately after it, so the caller can
 * time that one kernel. Pass NULL to clear. Process-wide, not thread-safe; the
 * main kernel is the tensor-core (or SIMT) attention kernel for GBS_OP_FWD and
 * GBS_OP_BWD and the split kernel for GBS_OP_DECODE. */
GBS_API gbs_status gbs_set_timer(int op, void* start, void* stop);

/* Total number of CUDA kernels this library has launched in this process. */
GBS_API uint64_t gbs_launch_count(void);

/* Failure-detection self-test (no counterpart in the paper). Launches one
 * thread that waits, through the same bounded mbarrier wait every pipeline
 * stage of the tensor-core kernels uses, on a shared-memory barrier that
 * nothing arrives at. After limit_us microseconds (1 .. 1,000,000) the wait
 * gives up, GBS_ERR_TIMEOUT is recorded in the error word of `ws` (its first
 * 4 bytes; any device buffer of at least 256 bytes, 256-byte aligned) and the
 * kernel returns; gbs_check(ws, stream) then reports it. Nothing traps or
 * faults, so the CUDA context stays usable. Returns GBS_ERR_WORKSPACE or
 * GBS_ERR_INVALID_ARG for a bad `ws` or limit, GBS_ERR_CUDA if the launch
 * fails. */
GBS_API gbs_status gbs_selftest_wait_timeout(void* ws, unsigned int limit_us, void* stream);

/* Bytes of device scratch that gbs_decode_noalloc keeps in the library. */
#define GBS_DECODE_NOALLOC_SCRATCH_BYTES (8u << 20)

/* Sparse decode without a workspace (no counterpart in the paper: this is a
 * convenience of this library, not part of the method).
 * Same inputs, outputs and results as gbs_decode, for callers that cannot
 * allocate device memory when they decode, e.g. a serving loop whose device
 * memory is reserved up front by another allocator, or one that must not call
 * cudaMalloc on its hot path because that call can synchronise the device.
 * The Top-K lists and per-split partials live in a static device array of
 * GBS_DECODE_NOALLOC_SCRATCH_BYTES that every GPU loading the library holds
 * until the process exits. The first call on each device looks up that
 * array's address (cudaGetSymbolAddress, with the device current); make that
 * first call before any stream capture. Calls on one device share the array:
 * calls that overlap on the GPU race and must be serialised by the caller.
 * Validates its arguments exactly as gbs_decode does (same statuses). With
 * num_splits = 0 it picks gbs_decode's split count, and so returns bitwise the
 * same results, unless those partials would not fit the array, in which case
 * it takes the largest count that fits. Rejects, with GBS_ERR_INVALID_ARG and a
 * gbs_last_error() message, any size whose scratch (about
 * B*Hq*(8*topk + 8 + splits*(4*d + 8)) bytes, splits <= 32) exceeds the array;
 * allocates and frees nothing. */
GBS_API gbs_status gbs_decode_noalloc(const gbs_params* p, const void* q, const void* Kc,
                                      const void* Vc, const float* S, void* O, float* LSE,
                                      int num_splits, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* GBS_H_ */
