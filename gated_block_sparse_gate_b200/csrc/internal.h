// internal.h — launchers shared between the C ABI (gbs_api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "gbs.h"

namespace gbs {

// Bookkeeping shared by all launchers: every kernel launch is counted, and
// the main kernel of an op is bracketed by the caller's timer events if set.
void note_launch(int n = 1);
// Sets the text returned by gbs_last_error() on the calling thread.
void set_last_error(const char* msg);
void timer_begin(int op, cudaStream_t st);
void timer_end(int op, cudaStream_t st);

// Resolved problem description handed to every launcher.
struct Problem {
  int B, Hq, Hkv, N, d, bs, Nb, G, topk, mode, dtype;
  float scale;        // logit scale (natural units)
  float scale_log2;   // scale * log2(e)
  float log_tau;      // threshold mode: ln(tau); 0 otherwise
};

// Validates a parameter block for one op (GBS_OP_FWD / BWD / DECODE) and
// resolves it; on failure sets gbs_last_error() and returns the status.
gbs_status resolve_params(const gbs_params* in, int op, Problem* out);
// Most decode splits a call can ask for.
constexpr int kMaxDecodeSplits = 32;
// The decode's automatic split count for n_ent blocks per selection row:
// the larger of "at most 17 blocks per CTA" and "two waves of resident CTAs",
// clamped to [1, min(n_ent, kMaxDecodeSplits)].
cudaError_t decode_auto_splits(const Problem& p, bool grouped, int n_ent, int* splits);

// Selection buffers produced by K1 and read by the attention kernels.
struct Selection {
  float* slse;     // [B, Hq, Nb]   training normaliser (may be null in sparse mode)
  int32_t* idx;    // [B, Hq, Nb, topk] (sparse only)
  int32_t* cnt;    // [B, Hq, Nb]
  float* logg;     // [B, Hq, Nb, topk]
};

// K1: gate normalisation (+ Top-K in sparse and threshold modes; `mode` is a
// gbs_mode, `log_tau` = ln(tau) is read in threshold mode only).
// rows_per_head = Nb for prefill/training (row r has history r); for decode
// rows_per_head = 1 and every row has history `decode_cur`. Sparse and
// threshold modes can also write sel_lse [rows] (the log-sum-exp of S over
// the kept blocks) and mbits [rows, mwords] (bit c of word c/32 set when block
// c is kept; every word written).
// Decode with per-sequence lengths: pass seq_lens [B] (row b holds
// rows_per_seq consecutive rows; lengths are clamped to [1, max_len]) and
// decode_cur = -1.
struct SeqLens {
  const int32_t* lens = nullptr;
  int rows_per_seq = 1;
  int max_len = 0;
};
cudaError_t launch_select(const float* S, int n_rows, int row_stride, int rows_per_head,
                          int decode_cur, int topk, int mode, float log_tau, int32_t* idx,
                          int32_t* cnt, float* logg, float* slse, cudaStream_t st,
                          float* sel_lse = nullptr, uint32_t* mbits = nullptr, int mwords = 0,
                          SeqLens seq = SeqLens());

// Exact SIMT path (fp32 math for fp32 or bf16 storage).
cudaError_t launch_fwd_simt(const Problem& p, const void* Q, const void* K, const void* V,
                            const float* S, const Selection& sel, void* O, float* LSE,
                            cudaStream_t st);
cudaError_t launch_bwd_simt(const Problem& p, const void* Q, const void* K, const void* V,
                            const float* S, const float* slse, const void* O, const float* LSE,
                            const void* dO, void* dQ, void* dK, void* dV, float* dS,
                            float* Dvec, float* Gblk, const uint32_t* mbits, int mwords,
                            cudaStream_t st);

// Where the decode finds a sequence's cache: contiguous [B, Hkv, N, d] (btab
// null) or pages [num_pages, Hkv, 64, d] through btab [B, max_blocks]; every
// sequence has length N (seq_lens null) or seq_lens[b]. Out-of-range pages or
// lengths are skipped / clamped on the device and reported in *err.
struct KvLayout {
  const int32_t* btab = nullptr;
  int max_blocks = 0, num_pages = 0;
  const int32_t* seq_lens = nullptr;
  unsigned int* err = nullptr;
};

// Decode (split over the selected blocks, then combine). With `grouped` the
// selection rows are [B, Hkv] and every q-head of a group uses its group's.
cudaError_t launch_decode(const Problem& p, const void* q, const void* Kc, const void* Vc,
                          const Selection& sel, int num_splits, float* part_ml, float* part_acc,
                          void* O, float* LSE, cudaStream_t st, const KvLayout& kv, bool grouped);
// q-heads one decode CTA serves (they share a selection and a kv head).
int decode_heads_per_cta(const Problem& p, bool grouped);
// Decode split CTAs resident per SM for this configuration.
int decode_resident_ctas(const Problem& p, bool grouped);

// Tensor-core path (sm_100a, bf16). Returns cudaErrorNotSupported when the
// configuration is outside what the kernel handles.
cudaError_t launch_fwd_tc(const Problem& p, const void* Q, const void* K, const void* V,
                          const float* S, const Selection& sel, const int32_t* plan,
                          int plan_stride, void* O, float* LSE, unsigned int* err,
                          cudaStream_t st);
bool fwd_tc_supported(const Problem& p);
// Training mode with an even q-heads-per-kv-head ratio: two query tiles per CTA.
cudaError_t launch_fwd_tc2(const Problem& p, const void* Q, const void* K, const void* V,
                           const float* S, const float* slse, void* O, float* LSE,
                           unsigned int* err, cudaStream_t st);
bool fwd_tc2_supported(const Problem& p);
// Per-(batch, head, 128-row tile) slot plan of sparse mode (union of the tile's
// two query blocks' Top-K lists plus their current blocks, with per-half biases).
cudaError_t launch_plan(const Problem& p, const Selection& sel, int32_t* plan, int plan_stride,
                        int n_tiles, cudaStream_t st);
// Backward. `slse` is the gate normaliser (over H_r in training mode, over the
// kept blocks otherwise); outside training mode `mbits` is K1's kept-block
// bitmap and `plan` a workspace of bwd_plan_ints(p) ints where the launcher
// lists, per (batch, kv-head, 128-key tile), the (q-head, 128-query tile)
// steps that touch a kept block.
cudaError_t launch_bwd_tc(const Problem& p, const void* Q, const void* K, const void* V,
                          const float* S, const float* slse, const void* O, const float* LSE,
                          const void* dO, void* dQ, void* dK, void* dV, float* Dvec, float* Gblk,
                          float* dQacc, const uint32_t* mbits, int mwords, int32_t* plan,
                          unsigned int* err, cudaStream_t st);
bool bwd_tc_supported(const Problem& p);
size_t bwd_plan_ints(const Problem& p);
// dS from the tile sums G (shared by both backward paths); mbits as above.
cudaError_t launch_ds_finalize(const Problem& p, const float* S, const float* slse,
                               const float* Gblk, float* dS, const uint32_t* mbits, int mwords,
                               cudaStream_t st);

}  // namespace gbs
