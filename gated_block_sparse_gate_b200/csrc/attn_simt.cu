// attn_simt.cu — exact fp32 SIMT path of the gated attention (forward and
// backward).
//
// Logit of query i and key j: z_ij = scale * q_i.k_j + b_ij, where b_ij is the
// normalised log gate of key block c(j) for query block r(i) when c(j) is an
// attended historical block, 0 for the always-kept current block with j <= i,
// and -inf otherwise (ai.viyan.live, "SAS Learns Token Importance for Sparse
// Attention", "The Logit Injection Mechanism"; HF paper page of "SAS: Simple
// Attention Sparsification via End-to-End Optimization of Context Ranking",
// Abstract). Training mode attends every earlier block (NeurIPS 2026 poster
// page, Abstract); sparse mode the Top-K list produced by K1. The backward
// reads the normaliser `nlse` (over H_r in training mode, over the kept blocks
// A_r otherwise) and, outside training mode, the kept-block bitmap of K1: a
// block outside A_r is skipped and its tile sum G is 0. The selection itself
// is a discrete choice and passes no gradient; dS flows through the
// renormalised gates of the kept blocks only.
//
// This path computes in fp32 on the CUDA cores with one thread per query (or
// key) row and a 64-row block per CTA. It serves fp32 inputs, where tensor-core
// tf32 cannot meet a 1e-5 tolerance, and any shape the tensor-core kernels do
// not handle. Everything is exact up to fp32 rounding; exp2 works in the log2
// domain with log2(e) folded into the scale and the bias.
#include "common.cuh"
#include "internal.h"

namespace gbs {

namespace {

constexpr int kBS = 64;  // context-unit block size this path supports

// Whether block c is kept for score row `row` (always, without a bitmap).
__device__ __forceinline__ bool kept(const uint32_t* mbits, int mwords, size_t row, int c) {
  return !mbits || ((__ldg(mbits + row * mwords + (c >> 5)) >> (c & 31)) & 1u);
}

template <typename T, int D>
__device__ __forceinline__ void load_rows(float* dst, int ld, const T* src, int tid, int nthr) {
  for (int e = tid; e < kBS * D; e += nthr) {
    const int row = e / D, col = e - row * D;
    dst[row * ld + col] = to_f32<T>(src[(size_t)row * D + col]);
  }
}

// ---------------------------------------------------------------- forward

template <typename T, int D>
__global__ void __launch_bounds__(kBS)
fwd_simt_kernel(Problem p, const T* __restrict__ Q, const T* __restrict__ K,
                const T* __restrict__ V, const float* __restrict__ S, Selection sel,
                T* __restrict__ O, float* __restrict__ LSE) {
  extern __shared__ float smem[];
  float* Qs = smem;                 // [64][D+1]
  float* Ks = Qs + kBS * (D + 1);   // [64][D]
  float* Vs = Ks + kBS * D;         // [64][D]
  const int r = blockIdx.x, h = blockIdx.y, b = blockIdx.z, t = threadIdx.x;
  const int kvh = h / p.G;
  const size_t qbase = ((size_t)(b * p.Hq + h) * p.N) * D;
  const size_t kvbase = ((size_t)(b * p.Hkv + kvh) * p.N) * D;
  const size_t row_id = (size_t)(b * p.Hq + h) * p.Nb + r;
  const bool train = p.mode == GBS_TRAIN;

  load_rows<T, D>(Qs, D + 1, Q + qbase + (size_t)r * kBS * D, t, kBS);
  const int nh = train ? r : sel.cnt[row_id];
  float m = -INFINITY, l = 0.f;
  float acc[D];
#pragma unroll
  for (int k = 0; k < D; ++k) acc[k] = 0.f;

  for (int a = 0; a <= nh; ++a) {
    int c;
    float bias;
    const bool diag = a == nh;
    if (diag) {
      c = r;
      bias = 0.f;
    } else if (train) {
      c = a;
      bias = S[row_id * p.Nb + c] - sel.slse[row_id];
    } else {
      c = sel.idx[row_id * p.topk + a];
      bias = sel.logg[row_id * p.topk + a];
    }
    __syncthreads();
    load_rows<T, D>(Ks, D, K + kvbase + (size_t)c * kBS * D, t, kBS);
    load_rows<T, D>(Vs, D, V + kvbase + (size_t)c * kBS * D, t, kBS);
    __syncthreads();
    const float bias2 = bias * GBS_LOG2E;
    const int jend = diag ? t + 1 : kBS;
    for (int j = 0; j < jend; ++j) {
      float s = 0.f;
#pragma unroll 16
      for (int k = 0; k < D; ++k) s = fmaf(Qs[t * (D + 1) + k], Ks[j * D + k], s);
      s = fmaf(s, p.scale_log2, bias2);
      if (s > m) {
        const float corr = exp2f(m - s);
        l *= corr;
#pragma unroll
        for (int k = 0; k < D; ++k) acc[k] *= corr;
        m = s;
      }
      const float pj = exp2f(s - m);
      l += pj;
#pragma unroll
      for (int k = 0; k < D; ++k) acc[k] = fmaf(pj, Vs[j * D + k], acc[k]);
    }
  }
  const float inv = 1.f / l;
  T* orow = O + qbase + (size_t)(r * kBS + t) * D;
#pragma unroll
  for (int k = 0; k < D; ++k) orow[k] = from_f32<T>(acc[k] * inv);
  LSE[(size_t)(b * p.Hq + h) * p.N + r * kBS + t] = (m + log2f(l)) * GBS_LN2;
}

// ---------------------------------------------------------------- backward

// D_i = sum_d dO_i * O_i, one warp per row.
template <typename T, int D>
__global__ void bwd_dot_kernel(const T* __restrict__ O, const T* __restrict__ dO,
                               float* __restrict__ Dvec, size_t rows) {
  const size_t row = (size_t)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  float s = 0.f;
  for (int k = lane; k < D; k += 32)
    s += to_f32<T>(O[row * D + k]) * to_f32<T>(dO[row * D + k]);
  s = warp_sum(s);
  if (lane == 0) Dvec[row] = s;
}

// dQ for one query block (one thread per query row) plus the tile sums
// G[r, c] = sum over the (r, c) tile of dL/dz.
template <typename T, int D>
__global__ void __launch_bounds__(kBS)
bwd_dq_kernel(Problem p, const T* __restrict__ Q, const T* __restrict__ K,
              const T* __restrict__ V, const float* __restrict__ S,
              const float* __restrict__ slse, const float* __restrict__ LSE,
              const T* __restrict__ dO, const float* __restrict__ Dvec, T* __restrict__ dQ,
              float* __restrict__ Gblk, const uint32_t* __restrict__ mbits, int mwords) {
  extern __shared__ float smem[];
  float* Qs = smem;                   // [64][D+1]
  float* dOs = Qs + kBS * (D + 1);    // [64][D+1]
  float* Ks = dOs + kBS * (D + 1);    // [64][D]
  float* Vs = Ks + kBS * D;           // [64][D]
  __shared__ float red[2];
  const int r = blockIdx.x, h = blockIdx.y, b = blockIdx.z, t = threadIdx.x;
  const int kvh = h / p.G;
  const size_t qbase = ((size_t)(b * p.Hq + h) * p.N) * D;
  const size_t kvbase = ((size_t)(b * p.Hkv + kvh) * p.N) * D;
  const size_t row_id = (size_t)(b * p.Hq + h) * p.Nb + r;
  const size_t i = (size_t)(b * p.Hq + h) * p.N + r * kBS + t;

  load_rows<T, D>(Qs, D + 1, Q + qbase + (size_t)r * kBS * D, t, kBS);
  load_rows<T, D>(dOs, D + 1, dO + qbase + (size_t)r * kBS * D, t, kBS);
  const float lse2 = LSE[i] * GBS_LOG2E;
  const float Di = Dvec[i];
  float dq[D];
#pragma unroll
  for (int k = 0; k < D; ++k) dq[k] = 0.f;

  for (int c = 0; c <= r; ++c) {
    const bool diag = c == r;
    if (!diag && !kept(mbits, mwords, row_id, c)) {  // uniform over the CTA
      if (t == 0) Gblk[row_id * p.Nb + c] = 0.f;
      continue;
    }
    const float bias = diag ? 0.f : S[row_id * p.Nb + c] - slse[row_id];
    __syncthreads();
    load_rows<T, D>(Ks, D, K + kvbase + (size_t)c * kBS * D, t, kBS);
    load_rows<T, D>(Vs, D, V + kvbase + (size_t)c * kBS * D, t, kBS);
    __syncthreads();
    const float bias2 = bias * GBS_LOG2E;
    const int jend = diag ? t + 1 : kBS;
    float gsum = 0.f;
    for (int j = 0; j < jend; ++j) {
      float s = 0.f, dp = 0.f;
#pragma unroll 16
      for (int k = 0; k < D; ++k) {
        s = fmaf(Qs[t * (D + 1) + k], Ks[j * D + k], s);
        dp = fmaf(dOs[t * (D + 1) + k], Vs[j * D + k], dp);
      }
      const float pr = exp2f(fmaf(s, p.scale_log2, bias2) - lse2);
      const float dz = pr * (dp - Di);
      gsum += dz;
#pragma unroll
      for (int k = 0; k < D; ++k) dq[k] = fmaf(dz, Ks[j * D + k], dq[k]);
    }
    gsum = warp_sum(gsum);
    if ((t & 31) == 0) red[t >> 5] = gsum;
    __syncthreads();
    if (t == 0) Gblk[row_id * p.Nb + c] = red[0] + red[1];
  }
  T* out = dQ + qbase + (size_t)(r * kBS + t) * D;
#pragma unroll
  for (int k = 0; k < D; ++k) out[k] = from_f32<T>(dq[k] * p.scale);
}

// dK and dV for one key block of one kv-head, summed over the q-heads of the
// group. Two threads per key row, each accumulating half of the head dims.
template <typename T, int D>
__global__ void __launch_bounds__(2 * kBS)
bwd_dkdv_kernel(Problem p, const T* __restrict__ Q, const T* __restrict__ K,
                const T* __restrict__ V, const float* __restrict__ S,
                const float* __restrict__ slse, const float* __restrict__ LSE,
                const T* __restrict__ dO, const float* __restrict__ Dvec, T* __restrict__ dK,
                T* __restrict__ dV, const uint32_t* __restrict__ mbits, int mwords) {
  constexpr int H2 = D / 2;
  extern __shared__ float smem[];
  float* Ks = smem;                    // [64][D+1] own key block
  float* Vs = Ks + kBS * (D + 1);      // [64][D+1]
  float* Qs = Vs + kBS * (D + 1);      // [64][D]   query block
  float* dOs = Qs + kBS * D;           // [64][D]
  float* lse2s = dOs + kBS * D;        // [64]
  float* Ds = lse2s + kBS;             // [64]
  const int c = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z, t = threadIdx.x;
  const int j = t & (kBS - 1), half = t >> 6;
  const size_t kvbase = ((size_t)(b * p.Hkv + kvh) * p.N) * D;
  load_rows<T, D>(Ks, D + 1, K + kvbase + (size_t)c * kBS * D, t, 2 * kBS);
  load_rows<T, D>(Vs, D + 1, V + kvbase + (size_t)c * kBS * D, t, 2 * kBS);
  float dk[H2], dv[H2];
#pragma unroll
  for (int k = 0; k < H2; ++k) dk[k] = dv[k] = 0.f;

  for (int hh = 0; hh < p.G; ++hh) {
    const int h = kvh * p.G + hh;
    const size_t qbase = ((size_t)(b * p.Hq + h) * p.N) * D;
    for (int r = c; r < p.Nb; ++r) {
      const size_t row_id = (size_t)(b * p.Hq + h) * p.Nb + r;
      const bool diag = r == c;
      if (!diag && !kept(mbits, mwords, row_id, c)) continue;  // uniform over the CTA
      const float bias2 = (diag ? 0.f : S[row_id * p.Nb + c] - slse[row_id]) * GBS_LOG2E;
      __syncthreads();
      load_rows<T, D>(Qs, D, Q + qbase + (size_t)r * kBS * D, t, 2 * kBS);
      load_rows<T, D>(dOs, D, dO + qbase + (size_t)r * kBS * D, t, 2 * kBS);
      if (t < kBS) {
        const size_t ii = (size_t)(b * p.Hq + h) * p.N + r * kBS + t;
        lse2s[t] = LSE[ii] * GBS_LOG2E;
        Ds[t] = Dvec[ii];
      }
      __syncthreads();
      for (int i = diag ? j : 0; i < kBS; ++i) {
        float s = 0.f, dp = 0.f;
#pragma unroll 16
        for (int k = 0; k < D; ++k) {
          s = fmaf(Qs[i * D + k], Ks[j * (D + 1) + k], s);
          dp = fmaf(dOs[i * D + k], Vs[j * (D + 1) + k], dp);
        }
        const float pr = exp2f(fmaf(s, p.scale_log2, bias2) - lse2s[i]);
        const float dz = pr * (dp - Ds[i]);
#pragma unroll
        for (int k = 0; k < H2; ++k) {
          dv[k] = fmaf(pr, dOs[i * D + half * H2 + k], dv[k]);
          dk[k] = fmaf(dz, Qs[i * D + half * H2 + k], dk[k]);
        }
      }
    }
  }
  const size_t orow = kvbase + (size_t)(c * kBS + j) * D + half * H2;
#pragma unroll
  for (int k = 0; k < H2; ++k) {
    dK[orow + k] = from_f32<T>(dk[k] * p.scale);
    dV[orow + k] = from_f32<T>(dv[k]);
  }
}

// dS[r, c'] = G[r, c'] - g[r, c'] * sum_{c<r} G[r, c] for kept c' < r, else 0
// (G is 0 outside the kept set, so the sum runs over it).
__global__ void ds_finalize_kernel(const float* __restrict__ S, const float* __restrict__ slse,
                                   const float* __restrict__ Gblk, float* __restrict__ dS,
                                   int Nb, size_t rows, const uint32_t* __restrict__ mbits,
                                   int mwords) {
  const size_t row = (size_t)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const int r = (int)(row % Nb);
  const float* g = Gblk + row * Nb;
  float tot = 0.f;
  for (int c = lane; c < r; c += 32) tot += g[c];
  tot = warp_sum(tot);
  const float lse = slse[row];
  for (int c = lane; c < Nb; c += 32)
    dS[row * Nb + c] =
        (c < r && kept(mbits, mwords, row, c)) ? g[c] - expf(S[row * Nb + c] - lse) * tot : 0.f;
}

template <typename T, int D>
cudaError_t fwd_simt_typed(const Problem& p, const void* Q, const void* K, const void* V,
                           const float* S, const Selection& sel, void* O, float* LSE,
                           cudaStream_t st) {
  const size_t smem = sizeof(float) * (kBS * (D + 1) + 2 * kBS * D);
  auto kern = fwd_simt_kernel<T, D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(p.Nb, p.Hq, p.B);
  kern<<<grid, kBS, smem, st>>>(p, (const T*)Q, (const T*)K, (const T*)V, S, sel, (T*)O, LSE);
  note_launch();
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t bwd_simt_typed(const Problem& p, const void* Q, const void* K, const void* V,
                           const float* S, const float* slse, const void* O, const float* LSE,
                           const void* dO, void* dQ, void* dK, void* dV, float* dS, float* Dvec,
                           float* Gblk, const uint32_t* mbits, int mwords, cudaStream_t st) {
  const size_t rows = (size_t)p.B * p.Hq * p.N;
  bwd_dot_kernel<T, D><<<(unsigned)((rows + 7) / 8), 256, 0, st>>>((const T*)O, (const T*)dO,
                                                                   Dvec, rows);
  note_launch();
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  {
    const size_t smem = sizeof(float) * (2 * kBS * (D + 1) + 2 * kBS * D);
    auto kern = bwd_dq_kernel<T, D>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    timer_begin(GBS_OP_BWD, st);
    kern<<<dim3(p.Nb, p.Hq, p.B), kBS, smem, st>>>(p, (const T*)Q, (const T*)K, (const T*)V, S,
                                                    slse, LSE, (const T*)dO, Dvec, (T*)dQ, Gblk,
                                                    mbits, mwords);
    note_launch();
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  {
    const size_t smem = sizeof(float) * (2 * kBS * (D + 1) + 2 * kBS * D + 2 * kBS);
    auto kern = bwd_dkdv_kernel<T, D>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<dim3(p.Nb, p.Hkv, p.B), 2 * kBS, smem, st>>>(p, (const T*)Q, (const T*)K, (const T*)V,
                                                         S, slse, LSE, (const T*)dO, Dvec,
                                                         (T*)dK, (T*)dV, mbits, mwords);
    note_launch();
    timer_end(GBS_OP_BWD, st);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  const size_t srows = (size_t)p.B * p.Hq * p.Nb;
  ds_finalize_kernel<<<(unsigned)((srows + 7) / 8), 256, 0, st>>>(S, slse, Gblk, dS, p.Nb, srows,
                                                                  mbits, mwords);
  note_launch();
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_ds_finalize(const Problem& p, const float* S, const float* slse,
                               const float* Gblk, float* dS, const uint32_t* mbits, int mwords,
                               cudaStream_t st) {
  const size_t srows = (size_t)p.B * p.Hq * p.Nb;
  ds_finalize_kernel<<<(unsigned)((srows + 7) / 8), 256, 0, st>>>(S, slse, Gblk, dS, p.Nb, srows,
                                                                  mbits, mwords);
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_fwd_simt(const Problem& p, const void* Q, const void* K, const void* V,
                            const float* S, const Selection& sel, void* O, float* LSE,
                            cudaStream_t st) {
  if (p.bs != kBS) return cudaErrorNotSupported;
  if (p.dtype == GBS_F32) {
    if (p.d == 64) return fwd_simt_typed<float, 64>(p, Q, K, V, S, sel, O, LSE, st);
    if (p.d == 128) return fwd_simt_typed<float, 128>(p, Q, K, V, S, sel, O, LSE, st);
  } else {
    if (p.d == 64) return fwd_simt_typed<__nv_bfloat16, 64>(p, Q, K, V, S, sel, O, LSE, st);
    if (p.d == 128) return fwd_simt_typed<__nv_bfloat16, 128>(p, Q, K, V, S, sel, O, LSE, st);
  }
  return cudaErrorNotSupported;
}

cudaError_t launch_bwd_simt(const Problem& p, const void* Q, const void* K, const void* V,
                            const float* S, const float* slse, const void* O, const float* LSE,
                            const void* dO, void* dQ, void* dK, void* dV, float* dS,
                            float* Dvec, float* Gblk, const uint32_t* mbits, int mwords,
                            cudaStream_t st) {
  if (p.bs != kBS) return cudaErrorNotSupported;
#define GBS_BWD(T, DD)                                                                       \
  return bwd_simt_typed<T, DD>(p, Q, K, V, S, slse, O, LSE, dO, dQ, dK, dV, dS, Dvec, Gblk,   \
                               mbits, mwords, st)
  if (p.dtype == GBS_F32) {
    if (p.d == 64) GBS_BWD(float, 64);
    if (p.d == 128) GBS_BWD(float, 128);
  } else {
    if (p.d == 64) GBS_BWD(__nv_bfloat16, 64);
    if (p.d == 128) GBS_BWD(__nv_bfloat16, 128);
  }
#undef GBS_BWD
  return cudaErrorNotSupported;
}

}  // namespace gbs
