// select.cu — K1: gate normalisation and Top-K block selection.
//
// Normalised softmax gates in log form (Hugging Face paper page of "SAS: Simple
// Attention Sparsification via End-to-End Optimization of Context Ranking",
// Abstract; ai.viyan.live blog, section "Differentiable Budget Constraints"),
// and the fixed-budget hard Top-K used at inference (NeurIPS 2026 poster page,
// Abstract).
//
// One warp owns one score row. Training mode only needs the row's log-sum-exp
// over the historical blocks c < r. Sparse mode maps the scores to
// order-preserving 32-bit keys once (in shared memory), finds the K-th largest
// key by an 8-bit radix select (four histogram passes, most significant digit
// first, per-warp bins, a warp scan to locate the bin holding rank K), keeps
// every block above that key plus the lowest-index blocks equal to it,
// compacts them in ascending index order with ballots, and renormalises the
// log gates over the kept set. Comparisons are exact on the fp32 scores, so
// the index lists are bit-identical to any other exact implementation of the
// same ordering.
//
// Threshold mode (ai.viyan.live blog, section "Implementation and Efficiency":
// only blocks whose importance passes a threshold are computed) first counts
// the blocks whose training-mode log gate S[r,c] - lse_r reaches ln(tau); the
// blocks passing are the highest-scoring ones, so the row then runs the same
// Top-k with k = min(topk, that count).
//
// For the sparse backward the kernel can also emit, per row, the normaliser
// over the kept set (sel_lse) and a bitmap of the kept blocks (bit c of word
// c / 32, every word of the row written).
#include "common.cuh"
#include "internal.h"

namespace gbs {

namespace {

constexpr int kWarps = 4;
constexpr int kRowCache = 2048;  // scores cached in shared memory per warp

__device__ __forceinline__ float row_score(const float* srow, const uint32_t* cache, bool cached,
                                           int c) {
  return cached ? __uint_as_float(cache[c]) : __ldg(srow + c);
}

// Locates, among the 256 bins of `hist` (lane l holds bins 8l..8l+7), the bin
// holding the element of rank kk counted from the top, and the number of
// elements in higher bins.
__device__ __forceinline__ int find_bin(const uint32_t* hist, int kk, int lane, int* above_out) {
  int c[8];
  int sum = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    c[i] = (int)hist[8 * lane + i];
    sum += c[i];
  }
  int incl = sum;  // sum over lanes >= lane
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_down_sync(0xffffffffu, incl, o);
    if (lane + o < 32) incl += t;
  }
  const int excl = incl - sum;  // sum over lanes > lane (higher bins)
  const unsigned bal = __ballot_sync(0xffffffffu, excl < kk && kk <= incl);
  const int src = __ffs(bal) - 1;
  int bin = 0, above = 0;
  if (lane == src) {
    int acc = excl;
    for (int i = 7; i >= 0; --i) {
      if (acc + c[i] >= kk) {
        bin = 8 * lane + i;
        above = acc;
        break;
      }
      acc += c[i];
    }
  }
  bin = __shfl_sync(0xffffffffu, bin, src);
  *above_out = __shfl_sync(0xffffffffu, above, src);
  return bin;
}

__global__ void __launch_bounds__(kWarps * 32)
select_kernel(const float* __restrict__ S, int n_rows, int row_stride, int rows_per_head,
              int decode_cur, int topk, int mode, float log_tau, int32_t* __restrict__ idx,
              int32_t* __restrict__ cnt, float* __restrict__ logg, float* __restrict__ slse,
              float* __restrict__ sel_lse, uint32_t* __restrict__ mbits, int mwords,
              SeqLens seq) {
  __shared__ uint32_t cache_all[kWarps][kRowCache];
  __shared__ uint32_t hist_all[kWarps][256];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * kWarps + warp;
  if (row >= n_rows) return;
  int r = decode_cur >= 0 ? decode_cur : (row % rows_per_head);
  if (seq.lens) {  // decode with one length per sequence: history = its current block
    int L = __ldg(seq.lens + row / seq.rows_per_seq);
    L = L < 1 ? 1 : (L > seq.max_len ? seq.max_len : L);
    r = (L - 1) / 64;
  }
  const float* srow = S + (size_t)row * row_stride;
  uint32_t* cache = cache_all[warp];
  const bool cached = r <= kRowCache;
  if (cached)
    for (int c = lane; c < r; c += 32) cache[c] = __float_as_uint(__ldg(srow + c));
  __syncwarp();

  // Training-mode normaliser over all of H_r.
  const bool threshold = mode == GBS_THRESHOLD;
  float row_lse = -INFINITY;
  if (slse || threshold) {
    float m = -INFINITY;
    for (int c = lane; c < r; c += 32) m = fmaxf(m, row_score(srow, cache, cached, c));
    m = warp_max(m);
    float s = 0.f;
    for (int c = lane; c < r; c += 32) s += expf(row_score(srow, cache, cached, c) - m);
    s = warp_sum(s);
    row_lse = r > 0 ? m + logf(s) : -INFINITY;
    if (slse && lane == 0) slse[row] = row_lse;
  }
  if (mode == GBS_TRAIN) return;

  int k = min(topk, r);
  if (threshold && k > 0) {
    int n = 0;
    for (int c = lane; c < r; c += 32) n += (row_score(srow, cache, cached, c) - row_lse) >= log_tau;
    k = min(k, __reduce_add_sync(0xffffffffu, n));
  }
  int32_t* out_idx = idx + (size_t)row * topk;
  float* out_logg = logg + (size_t)row * topk;

  // Threshold T = the k-th largest key; need_eq = how many keys equal to T
  // (lowest indices first) complete the top k.
  uint32_t T = 0u;
  int need_eq = 0;
  if (k > 0 && k < r && cached) {
    // keys once, then four 8-bit digit passes
    for (int c = lane; c < r; c += 32) cache[c] = ordered_key(__uint_as_float(cache[c]));
    __syncwarp();
    uint32_t* hist = hist_all[warp];
    uint32_t prefix = 0u, mask = 0u;
    int kk = k;
#pragma unroll 1
    for (int shift = 24; shift >= 0; shift -= 8) {
#pragma unroll
      for (int i = 0; i < 8; ++i) hist[8 * lane + i] = 0u;
      __syncwarp();
      for (int c = lane; c < r; c += 32) {
        const uint32_t u = cache[c];
        if ((u & mask) == prefix) atomicAdd(&hist[(u >> shift) & 255u], 1u);
      }
      __syncwarp();
      int above;
      const int bin = find_bin(hist, kk, lane, &above);
      kk -= above;
      prefix |= (uint32_t)bin << shift;
      mask |= 255u << shift;
      __syncwarp();
    }
    T = prefix;
    need_eq = kk;
    // back to scores for the compaction and the gate normalisation below
    for (int c = lane; c < r; c += 32) {
      const uint32_t u = cache[c];
      cache[c] = (u & 0x80000000u) ? (u & 0x7fffffffu) : ~u;
    }
    __syncwarp();
  } else if (k > 0 && k < r) {
    for (int bit = 31; bit >= 0; --bit) {
      const uint32_t cand = T | (1u << bit);
      int n = 0;
      for (int c = lane; c < r; c += 32) n += ordered_key(row_score(srow, cache, cached, c)) >= cand;
      n = __reduce_add_sync(0xffffffffu, n);
      if (n >= k) T = cand;
    }
    int gt = 0;
    for (int c = lane; c < r; c += 32) gt += ordered_key(row_score(srow, cache, cached, c)) > T;
    gt = __reduce_add_sync(0xffffffffu, gt);
    need_eq = k - gt;
  }

  // Compact the kept blocks in ascending index order.
  int written = 0, eq_seen = 0;
  float m = -INFINITY;
  const uint32_t lanes_below = (1u << lane) - 1u;
  int base = 0;
  for (; base < r && written < k; base += 32) {
    const int c = base + lane;
    const bool valid = c < r;
    const float s = valid ? row_score(srow, cache, cached, c) : 0.f;
    const uint32_t u = ordered_key(s);
    const bool eq = valid && k < r && u == T;
    const uint32_t eq_mask = __ballot_sync(0xffffffffu, eq);
    const int eq_before = eq_seen + __popc(eq_mask & lanes_below);
    const bool keep = valid && (k >= r || u > T || (eq && eq_before < need_eq));
    eq_seen += __popc(eq_mask);
    const uint32_t keep_mask = __ballot_sync(0xffffffffu, keep);
    if (mbits && lane == 0) mbits[(size_t)row * mwords + (base >> 5)] = keep_mask;
    const int pos = written + __popc(keep_mask & lanes_below);
    if (keep) {
      out_idx[pos] = c;
      out_logg[pos] = s;  // raw score for now, normalised below
      m = fmaxf(m, s);
    }
    written += __popc(keep_mask);
  }
  __syncwarp();
  m = warp_max(m);
  float sum = 0.f;
  for (int j = lane; j < k; j += 32) sum += expf(out_logg[j] - m);
  sum = warp_sum(sum);
  const float lse = m + logf(sum);
  for (int j = lane; j < topk; j += 32) {
    if (j < k) {
      out_logg[j] = out_logg[j] - lse;
    } else {
      out_idx[j] = -1;
      out_logg[j] = 0.f;
    }
  }
  if (lane == 0) cnt[row] = k;
  if (sel_lse && lane == 0) sel_lse[row] = lse;
  if (mbits)
    for (int wi = (base >> 5) + lane; wi < mwords; wi += 32) mbits[(size_t)row * mwords + wi] = 0u;
}


// ------------------------------------------------------------------ decode rows
// Decode has few score rows (one per sequence and head or kv group) of up to a
// few thousand blocks, so one CTA of 256 threads takes one row: the row's keys
// sit in shared memory, the radix passes share one histogram, and the kept
// blocks are compacted in index order through two block-wide prefix sums (a
// thread owns a contiguous segment, so the lowest-index ties come first). The
// selection is the same as select_kernel's.
constexpr int kRowThreads = 256;
constexpr int kRowCacheCta = 8192;

__device__ __forceinline__ float key_score(uint32_t u) {
  return __uint_as_float((u & 0x80000000u) ? (u & 0x7fffffffu) : ~u);
}

// Block-wide exclusive prefix sum of one int per thread; *total gets the sum.
__device__ __forceinline__ int block_excl_scan(int v, int* scratch, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  __syncthreads();
  if (lane == 31) scratch[warp] = incl;
  __syncthreads();
  int wbase = 0, tot = 0;
  for (int w = 0; w < kRowThreads / 32; ++w) {
    if (w < warp) wbase += scratch[w];
    tot += scratch[w];
  }
  *total = tot;
  return wbase + incl - v;
}

__device__ __forceinline__ float block_max(float v, float* scratch) {
  v = warp_max(v);
  __syncthreads();
  if ((threadIdx.x & 31) == 0) scratch[threadIdx.x >> 5] = v;
  __syncthreads();
  float m = -INFINITY;
  for (int w = 0; w < kRowThreads / 32; ++w) m = fmaxf(m, scratch[w]);
  return m;
}

__device__ __forceinline__ float block_sum(float v, float* scratch) {
  v = warp_sum(v);
  __syncthreads();
  if ((threadIdx.x & 31) == 0) scratch[threadIdx.x >> 5] = v;
  __syncthreads();
  float s = 0.f;
  for (int w = 0; w < kRowThreads / 32; ++w) s += scratch[w];
  return s;
}

__global__ void __launch_bounds__(kRowThreads)
select_row_cta_kernel(const float* __restrict__ S, int row_stride, int decode_cur, int topk,
                      int mode, float log_tau, int32_t* __restrict__ idx,
                      int32_t* __restrict__ cnt, float* __restrict__ logg, SeqLens seq) {
  // r_max + 1 words, sized at launch: a 2,048-block row takes 8 KB, so more CTAs
  // fit on an SM than with a fixed 32 KB array (per-head decode call on 64 x 131072,
  // K = 32: 0.363 -> 0.359 ms)
  extern __shared__ uint32_t keys[];
  __shared__ uint32_t hist[256];
  __shared__ int iscr[32];
  __shared__ float fscr[32];
  __shared__ int s_bin, s_above, s_cnt;
  const int row = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int r = decode_cur;
  if (seq.lens) {
    int L = __ldg(seq.lens + row / seq.rows_per_seq);
    L = L < 1 ? 1 : (L > seq.max_len ? seq.max_len : L);
    r = (L - 1) / 64;
  }
  const float* srow = S + (size_t)row * row_stride;
  for (int c = tid; c < r; c += kRowThreads) keys[c] = ordered_key(__ldg(srow + c));
  __syncthreads();

  int k = min(topk, r);
  if (mode == GBS_THRESHOLD && k > 0) {
    float m = -INFINITY;
    for (int c = tid; c < r; c += kRowThreads) m = fmaxf(m, key_score(keys[c]));
    m = block_max(m, fscr);
    float s = 0.f;
    for (int c = tid; c < r; c += kRowThreads) s += expf(key_score(keys[c]) - m);
    const float lse = m + logf(block_sum(s, fscr));
    int n = 0;
    for (int c = tid; c < r; c += kRowThreads) n += (key_score(keys[c]) - lse) >= log_tau;
    int total;
    block_excl_scan(n, iscr, &total);
    k = min(k, total);
  }

  // T = the k-th largest key; need_eq keys equal to T (lowest indices) complete the top k
  uint32_t T = 0u;
  int need_eq = 0;
  if (k > 0 && k < r) {
    uint32_t prefix = 0u, mask = 0u;
    int kk = k;
    bool early = false;
#pragma unroll 1
    for (int shift = 24; shift >= 0; shift -= 8) {
      for (int i = tid; i < 256; i += kRowThreads) hist[i] = 0u;
      __syncthreads();
      for (int c = tid; c < r; c += kRowThreads) {
        const uint32_t u = keys[c];
        if ((u & mask) == prefix) atomicAdd(&hist[(u >> shift) & 255u], 1u);
      }
      __syncthreads();
      if (warp == 0) {
        int above;
        const int bin = find_bin(hist, kk, lane, &above);
        if (lane == 0) {
          s_bin = bin;
          s_above = above;
          s_cnt = (int)hist[bin];
        }
      }
      __syncthreads();
      kk -= s_above;
      prefix |= (uint32_t)s_bin << shift;
      mask |= 255u << shift;
      if (s_cnt == kk && prefix != 0u) {
        // every key of the bin is needed: the top k are exactly the keys >= prefix
        // (those above the bin and the whole bin), so no later pass can change them
        early = true;
        break;
      }
    }
    T = early ? prefix - 1u : prefix;
    need_eq = early ? 0 : kk;
  }

  // compaction: thread tid owns blocks [c0, c1) in index order
  const int seg = (r + kRowThreads - 1) / kRowThreads;
  const int c0 = min(r, tid * seg), c1 = min(r, c0 + seg);
  const bool all = k >= r;
  int gt = 0, eq = 0;
  if (k > 0 && !all)
    for (int c = c0; c < c1; ++c) {
      const uint32_t u = keys[c];
      gt += u > T;
      eq += u == T;
    }
  int total;
  const int eq_before = block_excl_scan(eq, iscr, &total);
  const int eq_quota = k == 0 || all ? 0 : max(0, min(eq, need_eq - eq_before));
  const int keep = k == 0 ? 0 : (all ? c1 - c0 : gt + eq_quota);
  int pos = block_excl_scan(keep, iscr, &total);
  int32_t* out_idx = idx + (size_t)row * topk;
  float* out_logg = logg + (size_t)row * topk;
  if (keep > 0) {
    int eq_seen = 0;
    for (int c = c0; c < c1; ++c) {
      const uint32_t u = keys[c];
      bool kp = all || u > T;
      if (!all && u == T) {
        kp = eq_seen < eq_quota;
        ++eq_seen;
      }
      if (kp) {
        out_idx[pos] = c;
        out_logg[pos] = key_score(u);  // raw score for now, normalised below
        ++pos;
      }
    }
  }
  __syncthreads();  // the kept scores are in global memory, visible to the block
  float m = -INFINITY;
  for (int j = tid; j < k; j += kRowThreads) m = fmaxf(m, out_logg[j]);
  m = block_max(m, fscr);
  float s = 0.f;
  for (int j = tid; j < k; j += kRowThreads) s += expf(out_logg[j] - m);
  const float lse = m + logf(block_sum(s, fscr));
  for (int j = tid; j < topk; j += kRowThreads) {
    if (j < k) {
      out_logg[j] = out_logg[j] - lse;
    } else {
      out_idx[j] = -1;
      out_logg[j] = 0.f;
    }
  }
  if (tid == 0) cnt[row] = k;
}

}  // namespace

cudaError_t launch_select(const float* S, int n_rows, int row_stride, int rows_per_head,
                          int decode_cur, int topk, int mode, float log_tau, int32_t* idx,
                          int32_t* cnt, float* logg, float* slse, cudaStream_t st,
                          float* sel_lse, uint32_t* mbits, int mwords, SeqLens seq) {
  if (n_rows <= 0) return cudaSuccess;
  // decode rows (one history length per row, outputs idx/cnt/logg only): one CTA per row
  const bool decode = decode_cur >= 0 || seq.lens;
  const int r_max = seq.lens ? (seq.max_len - 1) / 64 : decode_cur;
  if (decode && mode != GBS_TRAIN && !slse && !sel_lse && !mbits && r_max <= kRowCacheCta) {
    select_row_cta_kernel<<<n_rows, kRowThreads, (size_t)(r_max + 1) * sizeof(uint32_t), st>>>(
        S, row_stride, decode_cur, topk, mode, log_tau, idx, cnt, logg, seq);
    note_launch();
    return cudaGetLastError();
  }
  const int grid = (n_rows + kWarps - 1) / kWarps;
  select_kernel<<<grid, kWarps * 32, 0, st>>>(S, n_rows, row_stride, rows_per_head, decode_cur,
                                              topk, mode, log_tau, idx, cnt, logg, slse, sel_lse,
                                              mbits, mwords, seq);
  note_launch();
  return cudaGetLastError();
}

}  // namespace gbs
