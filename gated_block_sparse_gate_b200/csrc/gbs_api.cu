// gbs_api.cu — the C ABI declared in include/gbs.h: argument validation,
// workspace layout and kernel dispatch. No allocation, no synchronisation
// (except gbs_check), no host-side compute.
#include <atomic>
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include "common.cuh"
#include "internal.h"

using namespace gbs;

namespace {

std::atomic<unsigned long long> g_launches{0};
cudaEvent_t g_timer[3][2] = {};

thread_local char g_last_error[256] = "";

gbs_status fail(gbs_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return s;
}

gbs_status cuda_status(cudaError_t e, const char* where) {
  if (e == cudaSuccess) return GBS_OK;
  if (e == cudaErrorNotSupported) return fail(GBS_ERR_UNSUPPORTED, "%s: unsupported configuration", where);
  return fail(GBS_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

constexpr size_t kAlign = 256;
constexpr int kMaxSplits = kMaxDecodeSplits;
inline size_t up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// Workspace carving: [header | regions...], each region 256-byte aligned.
struct Carver {
  char* base;
  size_t off = kAlign;  // header: device error word
  template <typename T>
  T* take(size_t count) {
    T* p = base ? reinterpret_cast<T*>(base + off) : nullptr;
    off += up(count * sizeof(T));
    return p;
  }
};

struct FwdWs {
  Selection sel;
  int32_t* plan;
  size_t bytes;
};
struct BwdWs {
  float *slse, *Dvec, *Gblk, *dQacc;  // slse: gate normaliser (over H_r, or over A_r)
  Selection sel;                      // outside training mode: K1's lists
  uint32_t* mbits;                    // outside training mode: kept-block bitmap
  int32_t* plan;                      // outside training mode, tensor-core path: step lists
  size_t bytes;
};

inline int mask_words(const Problem& p) { return (p.Nb + 31) / 32; }
struct DecWs {
  Selection sel;
  float *part_ml, *part_acc;
  size_t bytes;
};

inline size_t plan_stride(const Problem& p) { return (size_t)(2 * p.topk + 4); }

FwdWs carve_fwd(const Problem& p, void* ws) {
  Carver c{(char*)ws};
  FwdWs w{};
  const size_t rows = (size_t)p.B * p.Hq * p.Nb;
  w.sel.slse = c.take<float>(rows);
  if (p.mode != GBS_TRAIN) {
    w.sel.idx = c.take<int32_t>(rows * p.topk);
    w.sel.cnt = c.take<int32_t>(rows);
    w.sel.logg = c.take<float>(rows * p.topk);
    const size_t tiles = (size_t)p.B * p.Hq * ((p.Nb + 1) / 2);
    w.plan = c.take<int32_t>(tiles * plan_stride(p) * 3);
  }
  w.bytes = c.off;
  return w;
}

BwdWs carve_bwd(const Problem& p, void* ws) {
  Carver c{(char*)ws};
  BwdWs w{};
  w.slse = c.take<float>((size_t)p.B * p.Hq * p.Nb);
  w.Dvec = c.take<float>((size_t)p.B * p.Hq * p.N);
  w.Gblk = c.take<float>((size_t)p.B * p.Hq * p.Nb * p.Nb);
  if (bwd_tc_supported(p)) w.dQacc = c.take<float>((size_t)p.B * p.Hq * p.N * p.d);
  if (p.mode != GBS_TRAIN) {
    const size_t rows = (size_t)p.B * p.Hq * p.Nb;
    w.sel.idx = c.take<int32_t>(rows * p.topk);
    w.sel.cnt = c.take<int32_t>(rows);
    w.sel.logg = c.take<float>(rows * p.topk);
    w.mbits = c.take<uint32_t>(rows * mask_words(p));
    if (bwd_tc_supported(p)) w.plan = c.take<int32_t>(bwd_plan_ints(p));
  }
  w.bytes = c.off;
  return w;
}

DecWs carve_dec(const Problem& p, void* ws) {
  Carver c{(char*)ws};
  DecWs w{};
  const size_t rows = (size_t)p.B * p.Hq;
  w.sel.idx = c.take<int32_t>(rows * p.topk);
  w.sel.cnt = c.take<int32_t>(rows);
  w.sel.logg = c.take<float>(rows * p.topk);
  w.part_ml = c.take<float>(rows * kMaxSplits * 2);
  w.part_acc = c.take<float>(rows * kMaxSplits * p.d);
  w.bytes = c.off;
  return w;
}

bool aligned16(const void* ptr) { return ((uintptr_t)ptr & 15u) == 0; }

// Validates the parameter block and resolves it into a Problem.
gbs_status resolve(const gbs_params* in, int op, Problem* out) {
  if (!in) return fail(GBS_ERR_INVALID_ARG, "params is NULL");
  const gbs_params& q = *in;
  if (q.B <= 0 || q.Hq <= 0 || q.Hkv <= 0 || q.N <= 0 || q.d <= 0 || q.block <= 0)
    return fail(GBS_ERR_INVALID_ARG, "B, Hq, Hkv, N, d and block must be positive");
  if (q.Hq % q.Hkv) return fail(GBS_ERR_INVALID_ARG, "Hq (%d) must be a multiple of Hkv (%d)", q.Hq, q.Hkv);
  if (q.mode != GBS_TRAIN && q.mode != GBS_SPARSE && q.mode != GBS_THRESHOLD)
    return fail(GBS_ERR_INVALID_ARG, "mode %d unknown", q.mode);
  if (q.mode == GBS_THRESHOLD && !(q.tau > 0.f && q.tau <= 1.f))
    return fail(GBS_ERR_INVALID_ARG, "threshold mode needs 0 < tau <= 1 (got %g)", (double)q.tau);
  if (q.dtype != GBS_BF16 && q.dtype != GBS_F32) return fail(GBS_ERR_INVALID_ARG, "dtype %d unknown", q.dtype);
  if (!(q.scale >= 0.f) || isinf(q.scale)) return fail(GBS_ERR_INVALID_ARG, "scale must be finite and >= 0");
  if (op != GBS_OP_FWD && op != GBS_OP_BWD && op != GBS_OP_DECODE)
    return fail(GBS_ERR_INVALID_ARG, "op %d unknown", op);
  const bool uses_topk = (op == GBS_OP_DECODE) || (q.mode != GBS_TRAIN);
  if (uses_topk && (q.topk < 0 || q.topk > GBS_MAX_TOPK))
    return fail(GBS_ERR_INVALID_ARG, "topk %d outside [0, %d]", q.topk, GBS_MAX_TOPK);
  if (op != GBS_OP_DECODE && q.N % q.block)
    return fail(GBS_ERR_INVALID_ARG, "N (%d) must be a multiple of block (%d)", q.N, q.block);
  if (q.block != 64) return fail(GBS_ERR_UNSUPPORTED, "block %d: only 64 is built", q.block);
  if (q.d != 64 && q.d != 128) return fail(GBS_ERR_UNSUPPORTED, "d %d: only 64 and 128 are built", q.d);
  const size_t Nb = ((size_t)q.N + q.block - 1) / q.block;
  if ((size_t)q.B * q.Hq * Nb * Nb > ((size_t)1 << 40) || (size_t)q.B * q.Hq * q.N * q.d > ((size_t)1 << 40))
    return fail(GBS_ERR_INVALID_ARG, "problem too large");
  // token rows are TMA coordinates and grid indices: signed 32-bit
  if ((size_t)q.B * q.Hq * q.N > (size_t)INT32_MAX)
    return fail(GBS_ERR_INVALID_ARG, "problem too large: B * Hq * N must be below 2^31");
  Problem& p = *out;
  p.B = q.B; p.Hq = q.Hq; p.Hkv = q.Hkv; p.N = q.N; p.d = q.d; p.bs = q.block;
  p.Nb = (int)Nb; p.G = q.Hq / q.Hkv; p.topk = uses_topk ? q.topk : 0;
  p.mode = q.mode;
  if (op == GBS_OP_DECODE && q.mode != GBS_THRESHOLD) p.mode = GBS_SPARSE;
  p.dtype = q.dtype;
  p.log_tau = p.mode == GBS_THRESHOLD ? logf(q.tau) : 0.f;
  p.scale = q.scale > 0.f ? q.scale : 1.0f / sqrtf((float)q.d);
  p.scale_log2 = p.scale * GBS_LOG2E;
  return GBS_OK;
}

gbs_status check_ptrs(int n, const void* const* ptrs, const char* const* names) {
  for (int i = 0; i < n; ++i) {
    if (!ptrs[i]) return fail(GBS_ERR_INVALID_ARG, "%s is NULL", names[i]);
    if (!aligned16(ptrs[i])) return fail(GBS_ERR_INVALID_ARG, "%s is not 16-byte aligned", names[i]);
  }
  return GBS_OK;
}

gbs_status check_ws(const void* ws, size_t have, size_t need) {
  if (!ws) return fail(GBS_ERR_WORKSPACE, "workspace is NULL (need %zu bytes)", need);
  if ((uintptr_t)ws % kAlign) return fail(GBS_ERR_WORKSPACE, "workspace is not 256-byte aligned");
  if (have < need) return fail(GBS_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", have, need);
  return GBS_OK;
}

unsigned int* err_word(void* ws) { return reinterpret_cast<unsigned int*>(ws); }

}  // namespace

namespace gbs {
void set_last_error(const char* msg) { snprintf(g_last_error, sizeof(g_last_error), "%s", msg); }
gbs_status resolve_params(const gbs_params* in, int op, Problem* out) { return resolve(in, op, out); }

cudaError_t decode_auto_splits(const Problem& p, bool grouped, int n_ent, int* splits) {
  // Shares of at most 17 blocks per CTA, and at least two waves of the split
  // kernel's resident CTAs. On the 64 x 131072, K = 32 decode both variants
  // are fastest at 2 splits (16-17 blocks a CTA): per q-head row 0.363 ms
  // against 0.375 / 0.373 ms at 1 / 3; per shared-selection row 0.175 ms
  // against 0.179 ms at 3 and 0.187 ms at 6.
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const int cta_rows = grouped ? p.B * p.Hkv * (p.G / decode_heads_per_cta(p, true)) : p.B * p.Hq;
  const int two_waves = 2 * sms * decode_resident_ctas(p, grouped);
  const int by_share = (n_ent + 16) / 17;
  const int by_waves = (two_waves + cta_rows - 1) / cta_rows;
  int s = by_share > by_waves ? by_share : by_waves;
  if (s > n_ent) s = n_ent;
  if (s > kMaxSplits) s = kMaxSplits;
  if (s < 1) s = 1;
  *splits = s;
  return cudaSuccess;
}
void note_launch(int n) { g_launches.fetch_add((unsigned long long)n, std::memory_order_relaxed); }
void timer_begin(int op, cudaStream_t st) {
  if (g_timer[op][0]) cudaEventRecord(g_timer[op][0], st);
}
void timer_end(int op, cudaStream_t st) {
  if (g_timer[op][1]) cudaEventRecord(g_timer[op][1], st);
}
}  // namespace gbs

extern "C" {

gbs_status gbs_set_timer(int op, void* start, void* stop) {
  if (op < GBS_OP_FWD || op > GBS_OP_DECODE) return fail(GBS_ERR_INVALID_ARG, "op %d unknown", op);
  if ((start == nullptr) != (stop == nullptr))
    return fail(GBS_ERR_INVALID_ARG, "set both timer events or neither");
  g_timer[op][0] = (cudaEvent_t)start;
  g_timer[op][1] = (cudaEvent_t)stop;
  return GBS_OK;
}

uint64_t gbs_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }


int gbs_version(void) { return (GBS_VERSION_MAJOR << 16) | GBS_VERSION_MINOR; }

const char* gbs_status_string(gbs_status s) {
  switch (s) {
    case GBS_OK: return "ok";
    case GBS_ERR_INVALID_ARG: return "invalid argument";
    case GBS_ERR_UNSUPPORTED: return "unsupported configuration";
    case GBS_ERR_CUDA: return "CUDA error";
    case GBS_ERR_TIMEOUT: return "device wait timed out";
    case GBS_ERR_WORKSPACE: return "workspace missing or too small";
    case GBS_ERR_DEVICE_CHECK: return "device index check failed (debug build)";
  }
  return "unknown status";
}

const char* gbs_last_error(void) { return g_last_error; }

size_t gbs_workspace_bytes(const gbs_params* in, int op) {
  Problem p{};
  if (resolve(in, op, &p) != GBS_OK) return 0;
  if (op == GBS_OP_FWD) return carve_fwd(p, nullptr).bytes;
  if (op == GBS_OP_BWD) return carve_bwd(p, nullptr).bytes;
  return carve_dec(p, nullptr).bytes;
}

gbs_status gbs_clear_error(void* ws, void* stream) {
  if (!ws) return fail(GBS_ERR_WORKSPACE, "workspace is NULL");
  return cuda_status(cudaMemsetAsync(ws, 0, sizeof(unsigned int), (cudaStream_t)stream),
                     "gbs_clear_error");
}

gbs_status gbs_check(const void* ws, void* stream) {
  if (!ws) return fail(GBS_ERR_WORKSPACE, "workspace is NULL");
  unsigned int word = 0;
  cudaError_t e = cudaMemcpyAsync(&word, ws, sizeof(word), cudaMemcpyDeviceToHost, (cudaStream_t)stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_status(e, "gbs_check");
  if (word == 0) return GBS_OK;
  return fail((gbs_status)word, "device reported status %u", word);
}

gbs_status gbs_select(const gbs_params* in, const float* S, int32_t* idx, int32_t* cnt,
                      float* logg, float* slse, void* stream) {
  g_last_error[0] = 0;
  Problem p{};
  gbs_status s = resolve(in, GBS_OP_FWD, &p);
  if (s != GBS_OK) return s;
  const bool sparse = p.mode != GBS_TRAIN;
  if (!S) return fail(GBS_ERR_INVALID_ARG, "S is NULL");
  if (sparse && p.topk > 0 && (!idx || !logg)) return fail(GBS_ERR_INVALID_ARG, "idx/logg are NULL");
  if (sparse && !cnt) return fail(GBS_ERR_INVALID_ARG, "cnt is NULL");
  if (!sparse && !slse) return fail(GBS_ERR_INVALID_ARG, "slse is NULL in training mode");
  const int rows = p.B * p.Hq * p.Nb;
  return cuda_status(launch_select(S, rows, p.Nb, p.Nb, -1, p.topk, p.mode, p.log_tau, idx, cnt,
                                   logg, slse, (cudaStream_t)stream),
                     "gbs_select");
}

gbs_status gbs_fwd(const gbs_params* in, const void* Q, const void* K, const void* V,
                   const float* S, void* O, float* LSE, void* ws, size_t ws_bytes, void* stream) {
  g_last_error[0] = 0;
  Problem p{};
  gbs_status s = resolve(in, GBS_OP_FWD, &p);
  if (s != GBS_OK) return s;
  const void* ptrs[] = {Q, K, V, S, O, LSE};
  const char* names[] = {"Q", "K", "V", "S", "O", "LSE"};
  if ((s = check_ptrs(6, ptrs, names)) != GBS_OK) return s;
  FwdWs w = carve_fwd(p, nullptr);
  if ((s = check_ws(ws, ws_bytes, w.bytes)) != GBS_OK) return s;
  w = carve_fwd(p, ws);
  cudaStream_t st = (cudaStream_t)stream;
  const bool sparse = p.mode != GBS_TRAIN;
  const int rows = p.B * p.Hq * p.Nb;
  cudaError_t e = launch_select(S, rows, p.Nb, p.Nb, -1, p.topk, p.mode, p.log_tau, w.sel.idx,
                                w.sel.cnt, w.sel.logg, sparse ? nullptr : w.sel.slse, st);
  if (e != cudaSuccess) return cuda_status(e, "gbs_fwd/select");
  if (fwd_tc2_supported(p)) {
    e = launch_fwd_tc2(p, Q, K, V, S, w.sel.slse, O, LSE, err_word(ws), st);
    if (e != cudaErrorNotSupported) return cuda_status(e, "gbs_fwd/attention");
  }
  if (p.dtype == GBS_BF16 && fwd_tc_supported(p)) {
    e = launch_fwd_tc(p, Q, K, V, S, w.sel, w.plan, (int)plan_stride(p), O, LSE, err_word(ws), st);
    if (e != cudaErrorNotSupported) return cuda_status(e, "gbs_fwd/attention");
  }
  timer_begin(GBS_OP_FWD, st);
  e = launch_fwd_simt(p, Q, K, V, S, w.sel, O, LSE, st);
  timer_end(GBS_OP_FWD, st);
  return cuda_status(e, "gbs_fwd/attention");
}

gbs_status gbs_bwd(const gbs_params* in, const void* Q, const void* K, const void* V,
                   const float* S, const void* O, const float* LSE, const void* dO, void* dQ,
                   void* dK, void* dV, float* dS, void* ws, size_t ws_bytes, void* stream) {
  g_last_error[0] = 0;
  Problem p{};
  gbs_status s = resolve(in, GBS_OP_BWD, &p);
  if (s != GBS_OK) return s;
  const void* ptrs[] = {Q, K, V, S, O, LSE, dO, dQ, dK, dV, dS};
  const char* names[] = {"Q", "K", "V", "S", "O", "LSE", "dO", "dQ", "dK", "dV", "dS"};
  if ((s = check_ptrs(11, ptrs, names)) != GBS_OK) return s;
  BwdWs w = carve_bwd(p, nullptr);
  if ((s = check_ws(ws, ws_bytes, w.bytes)) != GBS_OK) return s;
  w = carve_bwd(p, ws);
  cudaStream_t st = (cudaStream_t)stream;
  const int rows = p.B * p.Hq * p.Nb;
  const int mwords = mask_words(p);
  cudaError_t e;
  if (p.mode == GBS_TRAIN)
    e = launch_select(S, rows, p.Nb, p.Nb, -1, 0, GBS_TRAIN, 0.f, nullptr, nullptr, nullptr,
                      w.slse, st);
  else  // the forward's selection, recomputed: normaliser over A_r and the kept bitmap
    e = launch_select(S, rows, p.Nb, p.Nb, -1, p.topk, p.mode, p.log_tau, w.sel.idx, w.sel.cnt,
                      w.sel.logg, nullptr, st, w.slse, w.mbits, mwords);
  if (e != cudaSuccess) return cuda_status(e, "gbs_bwd/select");
  if (bwd_tc_supported(p)) {
    e = launch_bwd_tc(p, Q, K, V, S, w.slse, O, LSE, dO, dQ, dK, dV, w.Dvec, w.Gblk, w.dQacc,
                      w.mbits, mwords, w.plan, err_word(ws), st);
    if (e == cudaSuccess) e = launch_ds_finalize(p, S, w.slse, w.Gblk, dS, w.mbits, mwords, st);
    return cuda_status(e, "gbs_bwd");
  }
  return cuda_status(launch_bwd_simt(p, Q, K, V, S, w.slse, O, LSE, dO, dQ, dK, dV, dS, w.Dvec,
                                     w.Gblk, w.mbits, mwords, st),
                     "gbs_bwd");
}

gbs_status gbs_decode(const gbs_params* in, const void* q, const void* Kc, const void* Vc,
                      const float* S, void* O, float* LSE, int num_splits, void* ws,
                      size_t ws_bytes, void* stream) {
  return gbs_decode_ex(in, nullptr, q, Kc, Vc, S, O, LSE, num_splits, ws, ws_bytes, stream);
}

gbs_status gbs_decode_ex(const gbs_params* in, const gbs_kv_layout* kvl, const void* q,
                         const void* Kc, const void* Vc, const float* S, void* O, float* LSE,
                         int num_splits, void* ws, size_t ws_bytes, void* stream) {
  g_last_error[0] = 0;
  Problem p{};
  gbs_status s = resolve(in, GBS_OP_DECODE, &p);
  if (s != GBS_OK) return s;
  const void* ptrs[] = {q, Kc, Vc, S, O, LSE};
  const char* names[] = {"q", "Kc", "Vc", "S", "O", "LSE"};
  if ((s = check_ptrs(6, ptrs, names)) != GBS_OK) return s;
  if (num_splits < 0 || num_splits > kMaxSplits)
    return fail(GBS_ERR_INVALID_ARG, "num_splits %d outside [0, %d]", num_splits, kMaxSplits);
  KvLayout kv;
  const bool grouped = kvl && kvl->group_shared;
  if (kvl) {
    if (kvl->group_shared != 0 && kvl->group_shared != 1)
      return fail(GBS_ERR_INVALID_ARG, "group_shared must be 0 or 1");
    if (kvl->block_table) {
      if (kvl->max_blocks < p.Nb)
        return fail(GBS_ERR_INVALID_ARG, "max_blocks (%d) is below ceil(N / block) = %d",
                    kvl->max_blocks, p.Nb);
      if (kvl->num_pages <= 0) return fail(GBS_ERR_INVALID_ARG, "num_pages must be positive");
      // a page's first cache row is a signed 32-bit index
      if ((size_t)kvl->num_pages * p.Hkv * p.bs > (size_t)INT32_MAX)
        return fail(GBS_ERR_INVALID_ARG, "num_pages * Hkv * block must be below 2^31");
      if ((uintptr_t)kvl->block_table & 3u)
        return fail(GBS_ERR_INVALID_ARG, "block_table is not 4-byte aligned");
    }
    if (kvl->seq_lens && ((uintptr_t)kvl->seq_lens & 3u))
      return fail(GBS_ERR_INVALID_ARG, "seq_lens is not 4-byte aligned");
    kv.btab = kvl->block_table;
    kv.max_blocks = kvl->max_blocks;
    kv.num_pages = kvl->num_pages;
    kv.seq_lens = kvl->seq_lens;
  }
  DecWs w = carve_dec(p, nullptr);
  if ((s = check_ws(ws, ws_bytes, w.bytes)) != GBS_OK) return s;
  w = carve_dec(p, ws);
  kv.err = err_word(ws);
  cudaStream_t st = (cudaStream_t)stream;
  const int sel_rows = grouped ? p.B * p.Hkv : p.B * p.Hq;  // one selection row each
  const int cur_max = (p.N - 1) / p.bs;
  SeqLens seq;
  seq.lens = kv.seq_lens;
  seq.rows_per_seq = grouped ? p.Hkv : p.Hq;
  seq.max_len = p.N;
  cudaError_t e = launch_select(S, sel_rows, p.Nb, 1, kv.seq_lens ? -1 : cur_max, p.topk, p.mode,
                                p.log_tau, w.sel.idx, w.sel.cnt, w.sel.logg, nullptr, st, nullptr,
                                nullptr, 0, seq);
  if (e != cudaSuccess) return cuda_status(e, "gbs_decode/select");
  const int n_ent = (p.topk < cur_max ? p.topk : cur_max) + 1;
  int splits = num_splits;
  if (splits == 0) {
    e = decode_auto_splits(p, grouped, n_ent, &splits);
    if (e != cudaSuccess) return cuda_status(e, "gbs_decode/splits");
  }
  if (splits > n_ent) splits = n_ent;
  if (splits > kMaxSplits) splits = kMaxSplits;
  if (splits < 1) splits = 1;
  return cuda_status(launch_decode(p, q, Kc, Vc, w.sel, splits, w.part_ml, w.part_acc, O, LSE, st,
                                   kv, grouped),
                     "gbs_decode");
}

}  // extern "C"
