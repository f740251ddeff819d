// fwd_tc2.cu — K2, training mode: gated flash-attention forward with two query
// tiles per CTA in ping-pong on the tcgen05 tensor cores (sm_100a).
//
// Same result as fwd_tc.cu (z_ij = scale q_i.k_j + b_ij with the normalised
// log gate of the historical key block, 0 with the causal mask on the current
// block; ai.viyan.live, "SAS Learns Token Importance for Sparse Attention",
// "The Logit Injection Mechanism"; HF paper page of "SAS: Simple Attention
// Sparsification via End-to-End Optimization of Context Ranking", Abstract),
// organised so the tensor cores never wait for one softmax:
//
//  * a CTA owns the same 128-row query tile of two q-heads (A, B) of one kv
//    group; in training mode both attend exactly the blocks 0..r, so every
//    K/V stage (two 64-key context blocks) is loaded once for both tiles;
//  * TMEM: S_A, S_B (128 fp32 columns each), O_A, O_B (128 each); P is written
//    back as bf16 over the first 64 columns of its S and fed to PV from TMEM;
//  * the MMA issuer interleaves PV_A(j), S_A(j+1), PV_B(j), S_B(j+1): while
//    softmax A works on S_A(j+1) the tensor cores run tile B's MMAs and vice
//    versa;
//  * softmax warps (one query row per thread) handle each 64-key slot with one
//    uniform code path (full gate bias, causal current block or masked): the
//    per-slot raw max comes first, then each logit costs one FFMA with the
//    slot constant (bias - running max) and one ex2;
//  * the O rescale is lazy (running max moves only when it grows by > 2^8);
//    O of a tile is quiescent whenever its next S has landed, because the
//    commit of that S covers the tile's previous PV.
// Warps: 0-3 softmax A, 4-7 softmax B, 8 TMA producer, 9 TMEM + MMA issuer.
// Every mbarrier wait is bounded and reports GBS_ERR_TIMEOUT.
#include <cuda.h>

#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace gbs {

namespace {

using namespace sm100;

constexpr int kBM = 128;
constexpr int kSlot = 64;
constexpr int kBN = 2 * kSlot;
constexpr int kThreads = 320;
constexpr int kTmemCols = 512;
constexpr uint64_t kTimeoutNs = 4000000000ull;
constexpr float kRescaleThreshold = 8.0f;
constexpr int kChunk = 128 * 128;  // 64 columns x 128 rows of bf16

template <int D>
struct Layout2 {
  static constexpr int kChunks = D / 64;
  static constexpr int kTile = kChunks * kChunk;
  static constexpr int kQAOff = 0;
  static constexpr int kQBOff = kTile;
  static constexpr int kKOff = 2 * kTile;  // two K stages
  static constexpr int kVOff = 4 * kTile;  // two V stages
  static constexpr int kBarOff = 6 * kTile;
  static constexpr int kSmemBytes = kBarOff + 256;
};

struct Bars2 {
  uint64_t q_full;
  uint64_t k_full[2], k_empty[2], v_full[2], v_empty[2];
  uint64_t s_full[2], p_full[2];
  uint64_t done;
  uint32_t tmem_base;
  int abort_flag;
};

struct Fwd2Args {
  Problem p;
  const float* S;
  const float* slse;
  int n_tiles;
  __nv_bfloat16* O;
  float* LSE;
  unsigned int* err;
};

enum : int { kMasked = 0, kDiag = 1, kFull = 2 };

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
__device__ __forceinline__ uint32_t cvt_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
fwd_tc2_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, Fwd2Args a) {
  using L = Layout2<D>;
  extern __shared__ __align__(1024) uint8_t smem[];
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0) set_error(a.err, GBS_ERR_UNSUPPORTED);
    return;
  }
  Bars2* bars = reinterpret_cast<Bars2*>(smem + L::kBarOff);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Problem& p = a.p;

  // CTA -> (tile, batch, head pair); heavy tiles first, consecutive CTAs share K/V
  const int pairs = p.B * (p.Hq / 2);
  const int tile = a.n_tiles - 1 - (int)(blockIdx.x / pairs);
  const int pr = (int)(blockIdx.x % pairs);
  const int b = pr / (p.Hq / 2), h0 = 2 * (pr % (p.Hq / 2));
  const int bhA = b * p.Hq + h0, bhB = bhA + 1;
  const int kvz = b * p.Hkv + h0 / p.G;
  const int n_stages = tile + 1;

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->k_empty[s], 1);
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->v_empty[s], 1);
      mbar_init(&bars->s_full[s], 1);
      mbar_init(&bars->p_full[s], 128);
    }
    mbar_init(&bars->done, 1);
    bars->abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 9) {
    tmem_alloc(&bars->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  volatile int* abort_flag = &bars->abort_flag;

  if (warp == 8) {
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      mbar_arrive_expect_tx(&bars->q_full, 2 * L::kTile);
      for (int ch = 0; ch < L::kChunks; ++ch) {
        tma_load_3d(smem + L::kQAOff + ch * kChunk, &tmQ, &bars->q_full, ch * 64, tile * kBM, bhA);
        tma_load_3d(smem + L::kQBOff + ch * kChunk, &tmQ, &bars->q_full, ch * 64, tile * kBM, bhB);
      }
      int issued = 0;
      for (int j = 0; j < n_stages; ++j) {
        const int st = j & 1;
        const int c0 = 2 * j, c1 = (2 * j + 1 < p.Nb) ? 2 * j + 1 : 0;
        if (j >= 2 && !mbar_wait(&bars->k_empty[st], ((j >> 1) - 1) & 1, abort_flag, a.err, kTimeoutNs))
          break;
        uint8_t* ks = smem + L::kKOff + st * L::kTile;
        mbar_arrive_expect_tx(&bars->k_full[st], L::kTile);
        for (int ch = 0; ch < L::kChunks; ++ch) {
          tma_load_3d(ks + ch * kChunk, &tmK, &bars->k_full[st], ch * 64, c0 * kSlot, kvz);
          tma_load_3d(ks + ch * kChunk + kSlot * 128, &tmK, &bars->k_full[st], ch * 64, c1 * kSlot, kvz);
        }
        if (j >= 2 && !mbar_wait(&bars->v_empty[st], ((j >> 1) - 1) & 1, abort_flag, a.err, kTimeoutNs))
          break;
        uint8_t* vs = smem + L::kVOff + st * L::kTile;
        mbar_arrive_expect_tx(&bars->v_full[st], L::kTile);
        for (int ch = 0; ch < L::kChunks; ++ch) {
          tma_load_3d(vs + ch * kChunk, &tmV, &bars->v_full[st], ch * 64, c0 * kSlot, kvz);
          tma_load_3d(vs + ch * kChunk + kSlot * 128, &tmV, &bars->v_full[st], ch * 64, c1 * kSlot, kvz);
        }
        issued = j + 1;
      }
      if (*abort_flag) {
        mbar_drain(&bars->q_full, 0, 1000000ull);
        for (int j = issued - 2 < 0 ? 0 : issued - 2; j < issued; ++j) {
          mbar_drain(&bars->k_full[j & 1], (j >> 1) & 1, 1000000ull);
          mbar_drain(&bars->v_full[j & 1], (j >> 1) & 1, 1000000ull);
        }
      }
    }
  } else if (warp == 9) {
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(kBM, kBN, 0);
      constexpr uint32_t idO = idesc_bf16_f32(kBM, D, 1);
      const uint32_t qa = smem_u32(smem + L::kQAOff), qb = smem_u32(smem + L::kQBOff);
      auto issue_s = [&](int x, int j) -> bool {
        const int st = j & 1;
        if (x == 0) {
          if (!mbar_wait(&bars->k_full[st], (j >> 1) & 1, abort_flag, a.err, kTimeoutNs)) return false;
          tc_fence_after();
        }
        const uint32_t q_addr = x ? qb : qa;
        const uint32_t k_addr = smem_u32(smem + L::kKOff + st * L::kTile);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const int ch = ks >> 2, kk = ks & 3;
          mma_ss(tmem + x * 128, sdesc_sw128(q_addr + ch * kChunk + kk * 32, 16, 1024),
                 sdesc_sw128(k_addr + ch * kChunk + kk * 32, 16, 1024), idS, ks > 0 ? 1u : 0u);
        }
        mma_commit(&bars->s_full[x]);
        if (x == 1) mma_commit(&bars->k_empty[st]);
        return true;
      };
      auto issue_pv = [&](int x, int j) -> bool {
        const int st = j & 1;
        if (!mbar_wait(&bars->p_full[x], j & 1, abort_flag, a.err, kTimeoutNs)) return false;
        if (x == 0 && !mbar_wait(&bars->v_full[st], (j >> 1) & 1, abort_flag, a.err, kTimeoutNs))
          return false;
        tc_fence_after();
        const uint32_t v_addr = smem_u32(smem + L::kVOff + st * L::kTile);
#pragma unroll
        for (int ks = 0; ks < kBN / 16; ++ks)
          mma_ts(tmem + 256 + x * 128, tmem + x * 128 + ks * 8,
                 sdesc_sw128(v_addr + ks * 2048, kChunk, 1024), idO, (j > 0 || ks > 0) ? 1u : 0u);
        if (x == 1) mma_commit(&bars->v_empty[st]);
        return true;
      };
      bool ok = mbar_wait(&bars->q_full, 0, abort_flag, a.err, kTimeoutNs);
      ok = ok && issue_s(0, 0) && issue_s(1, 0);
      for (int j = 0; ok && j < n_stages; ++j) {
        ok = issue_pv(0, j);
        if (ok && j + 1 < n_stages) ok = issue_s(0, j + 1);
        if (ok) ok = issue_pv(1, j);
        if (ok && j + 1 < n_stages) ok = issue_s(1, j + 1);
      }
      mma_commit(&bars->done);
      // after an abort the flag cuts the wait short: drain the MMAs still in
      // flight before tensor memory is freed
      if (!mbar_wait(&bars->done, 0, abort_flag, a.err, kTimeoutNs))
        mbar_drain(&bars->done, 0, 1000000ull);
    }
  } else {
    // ------------------------------------------------------------- softmax
    const int x = warp >> 2, quad = warp & 3;
    const int row = quad * 32 + lane;
    const int half = row >> 6, iloc = row & 63;
    const int myr = 2 * tile + half;
    const int bh = x ? bhB : bhA;
    const uint32_t tS = tmem + ((uint32_t)(quad * 32) << 16) + x * 128;
    const uint32_t tO = tS + 256;
    const float sc = p.scale_log2;
    const size_t srow = (size_t)bh * p.Nb + myr;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < n_stages; ++j) {
      int kind[2];
      float bias[2];
#pragma unroll
      for (int s = 0; s < 2; ++s) {
        const int c = 2 * j + s;
        kind[s] = kMasked;
        bias[s] = 0.f;
        if (myr < p.Nb && c <= myr) {
          if (c == myr) {
            kind[s] = kDiag;
          } else {
            kind[s] = kFull;
            bias[s] = (__ldg(a.S + srow * p.Nb + c) - __ldg(a.slse + srow)) * GBS_LOG2E;
          }
        }
      }
      if (!mbar_wait(&bars->s_full[x], j & 1, abort_flag, a.err, kTimeoutNs)) {
        ok = false;
        break;
      }
      tc_fence_after();
      // pass 1: per-slot maximum of the scaled, biased logits; slot 1 stays in
      // registers, slot 0 is read again in pass 2 (keeps register use low)
      uint32_t v1[64];
      float smax[2];
#pragma unroll
      for (int s = 0; s < 2; ++s) {
        uint32_t v[64];
        tmem_ld32(tS + s * 64, *reinterpret_cast<uint32_t(*)[32]>(v));
        tmem_ld32(tS + s * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(v + 32));
        tmem_wait_ld();
        if (kind[s] == kDiag) {
#pragma unroll
          for (int k = 0; k < 64; ++k)
            if (k > iloc) v[k] = __float_as_uint(-INFINITY);
        }
        float a0 = -INFINITY, a1 = -INFINITY, a2 = -INFINITY, a3 = -INFINITY;
#pragma unroll
        for (int k = 0; k < 64; k += 8) {
          a0 = max3(a0, __uint_as_float(v[k]), __uint_as_float(v[k + 1]));
          a1 = max3(a1, __uint_as_float(v[k + 2]), __uint_as_float(v[k + 3]));
          a2 = max3(a2, __uint_as_float(v[k + 4]), __uint_as_float(v[k + 5]));
          a3 = max3(a3, __uint_as_float(v[k + 6]), __uint_as_float(v[k + 7]));
        }
        const float raw = fmaxf(fmaxf(a0, a1), fmaxf(a2, a3));
        smax[s] = kind[s] == kMasked ? -INFINITY : fmaf(raw, sc, bias[s]);
        if (s == 1) {
#pragma unroll
          for (int k = 0; k < 64; ++k) v1[k] = v[k];
        }
      }
      const float mx = fmaxf(smax[0], smax[1]);
      const bool need = mx > m + kRescaleThreshold;
      if (__any_sync(0xffffffffu, need) && j > 0) {
        // O is quiescent: the commit that signalled this S covered the previous PV
        const float f = need ? ex2(m - mx) : 1.f;
#pragma unroll
        for (int q = 0; q < D / 32; ++q) {
          uint32_t o[32];
          tmem_ld32(tO + q * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * f);
          tmem_st32(tO + q * 32, o);
        }
        if (need) l *= f;
      }
      if (need) m = mx;
      const float mu = m == -INFINITY ? 0.f : m;
      float l0 = 0.f, l1 = 0.f, l2 = 0.f, l3 = 0.f;
      // pass 2, slot 0: 32-column chunks; bf16 P of keys [32c, 32c+32) goes to
      // columns [16c, 16c+16), which this pass has already read
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t pk[16];
        if (kind[0] == kMasked) {
#pragma unroll
          for (int k = 0; k < 16; ++k) pk[k] = 0u;
        } else {
          uint32_t v[32];
          tmem_ld32(tS + c * 32, v);
          tmem_wait_ld();
          const float cst = bias[0] - mu;
#pragma unroll
          for (int k = 0; k < 32; k += 4) {
            float x0 = fmaf(__uint_as_float(v[k]), sc, cst);
            float x1 = fmaf(__uint_as_float(v[k + 1]), sc, cst);
            float x2 = fmaf(__uint_as_float(v[k + 2]), sc, cst);
            float x3 = fmaf(__uint_as_float(v[k + 3]), sc, cst);
            if (kind[0] == kDiag) {
              const int kk = c * 32 + k;
              if (kk > iloc) x0 = -INFINITY;
              if (kk + 1 > iloc) x1 = -INFINITY;
              if (kk + 2 > iloc) x2 = -INFINITY;
              if (kk + 3 > iloc) x3 = -INFINITY;
            }
            const float p0 = ex2(x0), p1 = ex2(x1), p2 = ex2(x2), p3 = ex2(x3);
            l0 += p0;
            l1 += p1;
            l2 += p2;
            l3 += p3;
            pk[k / 2] = cvt_bf16x2(p0, p1);
            pk[k / 2 + 1] = cvt_bf16x2(p2, p3);
          }
        }
        tmem_st16(tS + c * 16, pk);
      }
      // slot 1 from registers -> columns [32, 64) (slot 0's upper half, read above)
      {
        uint32_t pk[32];
        if (kind[1] == kMasked) {
#pragma unroll
          for (int k = 0; k < 32; ++k) pk[k] = 0u;
        } else {
          const float cst = bias[1] - mu;
#pragma unroll
          for (int k = 0; k < 64; k += 4) {
            const float p0 = ex2(fmaf(__uint_as_float(v1[k]), sc, cst));
            const float p1 = ex2(fmaf(__uint_as_float(v1[k + 1]), sc, cst));
            const float p2 = ex2(fmaf(__uint_as_float(v1[k + 2]), sc, cst));
            const float p3 = ex2(fmaf(__uint_as_float(v1[k + 3]), sc, cst));
            l0 += p0;
            l1 += p1;
            l2 += p2;
            l3 += p3;
            pk[k / 2] = cvt_bf16x2(p0, p1);
            pk[k / 2 + 1] = cvt_bf16x2(p2, p3);
          }
        }
        tmem_st32(tS + 32, pk);
      }
      l += (l0 + l1) + (l2 + l3);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bars->p_full[x]);
    }
    if (ok && mbar_wait(&bars->done, 0, abort_flag, a.err, kTimeoutNs)) {
      tc_fence_after();
      const int qrow = tile * kBM + row;
      const bool valid = qrow < p.N;
      const float inv = 1.f / l;
      __nv_bfloat16* orow = a.O + ((size_t)bh * p.N + qrow) * D;
#pragma unroll
      for (int q = 0; q < D / 32; ++q) {
        uint32_t o[32];
        tmem_ld32(tO + q * 32, o);
        tmem_wait_ld();
        if (valid) {
          uint4* dst = reinterpret_cast<uint4*>(orow + q * 32);
#pragma unroll
          for (int k = 0; k < 4; ++k)
            dst[k] = make_uint4(cvt_bf16x2(__uint_as_float(o[8 * k]) * inv, __uint_as_float(o[8 * k + 1]) * inv),
                                cvt_bf16x2(__uint_as_float(o[8 * k + 2]) * inv, __uint_as_float(o[8 * k + 3]) * inv),
                                cvt_bf16x2(__uint_as_float(o[8 * k + 4]) * inv, __uint_as_float(o[8 * k + 5]) * inv),
                                cvt_bf16x2(__uint_as_float(o[8 * k + 6]) * inv, __uint_as_float(o[8 * k + 7]) * inv));
        }
      }
      if (valid) a.LSE[(size_t)bh * p.N + qrow] = (m + log2f(l)) * GBS_LN2;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

bool make_map2(CUtensorMap* m, const void* base, int d, int rows, int heads, int box_rows) {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return false;
    fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)rows, (cuuint64_t)heads};
  const cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)d * rows * 2};
  const cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D>
cudaError_t launch2(const Fwd2Args& a, const void* Q, const void* K, const void* V, cudaStream_t st) {
  const Problem& p = a.p;
  CUtensorMap tq, tk, tv;
  if (!make_map2(&tq, Q, D, p.N, p.B * p.Hq, kBM) || !make_map2(&tk, K, D, p.N, p.B * p.Hkv, kSlot) ||
      !make_map2(&tv, V, D, p.N, p.B * p.Hkv, kSlot))
    return cudaErrorInvalidValue;
  auto kern = fwd_tc2_kernel<D>;
  const int smem = Layout2<D>::kSmemBytes;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const unsigned grid = (unsigned)(p.B * (p.Hq / 2) * a.n_tiles);
  timer_begin(GBS_OP_FWD, st);
  kern<<<grid, kThreads, smem, st>>>(tq, tk, tv, a);
  timer_end(GBS_OP_FWD, st);
  note_launch();
  return cudaGetLastError();
}

}  // namespace

bool fwd_tc2_supported(const Problem& p) {
  return p.dtype == GBS_BF16 && p.mode == GBS_TRAIN && p.bs == kSlot && (p.d == 64 || p.d == 128) &&
         p.N % kSlot == 0 && p.G % 2 == 0;
}

cudaError_t launch_fwd_tc2(const Problem& p, const void* Q, const void* K, const void* V,
                           const float* S, const float* slse, void* O, float* LSE,
                           unsigned int* err, cudaStream_t st) {
  if (!fwd_tc2_supported(p)) return cudaErrorNotSupported;
  Fwd2Args a;
  a.p = p;
  a.S = S;
  a.slse = slse;
  a.n_tiles = (p.Nb + 1) / 2;
  a.O = reinterpret_cast<__nv_bfloat16*>(O);
  a.LSE = LSE;
  a.err = err;
  if (p.d == 64) return launch2<64>(a, Q, K, V, st);
  return launch2<128>(a, Q, K, V, st);
}

}  // namespace gbs
