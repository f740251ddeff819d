// fwd_tc2.cu — K2, training mode: gated flash-attention forward with two query
// tiles per CTA on the tcgen05 tensor cores (sm_100a).
//
// Same result as fwd_tc.cu (z_ij = scale q_i.k_j + b_ij with the normalised
// log gate of the historical key block, 0 with the causal mask on the current
// block; ai.viyan.live, "SAS Learns Token Importance for Sparse Attention",
// "The Logit Injection Mechanism"; HF paper page of "SAS: Simple Attention
// Sparsification via End-to-End Optimization of Context Ranking", Abstract),
// organised so that the tensor cores never wait for a softmax:
//
//  * a CTA owns the same 128-row query tile of two q-heads (A, B) of one kv
//    group; in training mode both attend exactly the blocks 0..r, so every
//    K/V stage (two 64-key context blocks) is loaded once for both tiles;
//  * TMEM: one 128-column S buffer that the two tiles take in turn, P_A and
//    P_B (64 columns each, bf16 pairs), O_A and O_B (128 each);
//  * a softmax copies its whole S tile into registers and releases the
//    buffer at once, so the next tile's S is computed while it works; the
//    MMA issuer runs S_A(j+1), PV_A(j), S_B(j+1), PV_B(j) and each S only
//    waits for the other tile's copy of the previous S, never for a P;
//  * softmax warps (one query row per thread, 208 registers after the
//    control warpgroup hands its registers over) take each 64-key slot with
//    one code path (full gate bias, causal current block or masked): the
//    slot's raw max first, then one FFMA with the slot constant
//    (bias - running max) and one ex2 per logit;
//  * the O rescale is lazy (the running max moves only when it grows by more
//    than 2^8); before it writes P a softmax waits for its tile's previous
//    PV, which also makes O quiescent for a rescale.
// Warps: 0-3 softmax A, 4-7 softmax B, 8 TMA producer, 9 TMEM + MMA issuer,
// 10-11 idle. Every mbarrier wait is bounded and reports GBS_ERR_TIMEOUT.
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
constexpr int kThreads = 384;
constexpr int kTmemCols = 512;
// registers per thread: 168 at launch (65536 / 384, rounded down to 8); the
// control warpgroup drops to 72 and the two softmax warpgroups rise to 208:
// 128 x (208 + 208 + 72) = 62464 <= 384 x 168 = 64512, and per sub-partition
// (one warp of each warpgroup) 32 x 488 = 15616 <= 16384
constexpr int kRegsSoftmax = 208;
constexpr int kRegsControl = 72;
static_assert(128 * (2 * kRegsSoftmax + kRegsControl) <= kThreads * 168, "register split");
constexpr uint64_t kTimeoutNs = 4000000000ull;
constexpr float kRescaleThreshold = 8.0f;
constexpr int kChunk = 128 * 128;  // 64 columns x 128 rows of bf16
// TMEM columns
constexpr uint32_t kColS = 0, kColP = 128, kColO = 256;

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
  uint64_t s_full[2], s_free[2], p_full[2], pv_done[2];  // [tile]
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
template <int N>
__device__ __forceinline__ void regs_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void regs_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
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
      mbar_init(&bars->s_free[s], 128);
      mbar_init(&bars->p_full[s], 128);
      mbar_init(&bars->pv_done[s], 1);
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

  if (warp >= 8) {
    regs_dec<kRegsControl>();
    if (warp == 8 && lane == 0) {
      // ---------------------------------------------------------- TMA producer
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
        // let loads still in flight land before the CTA exits
        mbar_drain(&bars->q_full, 0, 1000000ull);
        for (int j = issued - 2 < 0 ? 0 : issued - 2; j < issued; ++j) {
          mbar_drain(&bars->k_full[j & 1], (j >> 1) & 1, 1000000ull);
          mbar_drain(&bars->v_full[j & 1], (j >> 1) & 1, 1000000ull);
        }
      }
    } else if (warp == 9 && lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      constexpr uint32_t idS = idesc_bf16_f32(kBM, kBN, 0);
      constexpr uint32_t idO = idesc_bf16_f32(kBM, D, 1);
      const uint32_t qa = smem_u32(smem + L::kQAOff), qb = smem_u32(smem + L::kQBOff);
      // S_x(j) = Q_x K_j^T into the shared S buffer
      auto issue_s = [&](int x, int j) -> bool {
        const int st = j & 1;
        if (x == 0) {
          if (!mbar_wait(&bars->k_full[st], (j >> 1) & 1, abort_flag, a.err, kTimeoutNs)) return false;
        }
        // the buffer is free once the other tile has copied its previous S out
        if (!(x == 0 && j == 0) &&
            !mbar_wait(&bars->s_free[x ^ 1], (x ? j : j - 1) & 1, abort_flag, a.err, kTimeoutNs))
          return false;
        tc_fence_after();
        const uint32_t q_addr = x ? qb : qa;
        const uint32_t k_addr = smem_u32(smem + L::kKOff + st * L::kTile);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const int ch = ks >> 2, kk = ks & 3;
          mma_ss(tmem + kColS, sdesc_sw128(q_addr + ch * kChunk + kk * 32, 16, 1024),
                 sdesc_sw128(k_addr + ch * kChunk + kk * 32, 16, 1024), idS, ks > 0 ? 1u : 0u);
        }
        mma_commit(&bars->s_full[x]);
        if (x == 1) mma_commit(&bars->k_empty[st]);
        return true;
      };
      // O_x += P_x(j) V_j, P from its own TMEM columns
      auto issue_pv = [&](int x, int j) -> bool {
        const int st = j & 1;
        if (!mbar_wait(&bars->p_full[x], j & 1, abort_flag, a.err, kTimeoutNs)) return false;
        if (x == 0 && !mbar_wait(&bars->v_full[st], (j >> 1) & 1, abort_flag, a.err, kTimeoutNs))
          return false;
        tc_fence_after();
        const uint32_t v_addr = smem_u32(smem + L::kVOff + st * L::kTile);
#pragma unroll
        for (int ks = 0; ks < kBN / 16; ++ks)
          mma_ts(tmem + kColO + x * 128, tmem + kColP + x * 64 + ks * 8,
                 sdesc_sw128(v_addr + ks * 2048, kChunk, 1024), idO, (j > 0 || ks > 0) ? 1u : 0u);
        mma_commit(&bars->pv_done[x]);
        if (x == 1) mma_commit(&bars->v_empty[st]);
        return true;
      };
      bool ok = mbar_wait(&bars->q_full, 0, abort_flag, a.err, kTimeoutNs);
      ok = ok && issue_s(0, 0) && issue_s(1, 0);
      for (int j = 0; ok && j < n_stages; ++j) {
        if (j + 1 < n_stages) ok = issue_s(0, j + 1);
        if (ok) ok = issue_pv(0, j);
        if (ok && j + 1 < n_stages) ok = issue_s(1, j + 1);
        if (ok) ok = issue_pv(1, j);
      }
      mma_commit(&bars->done);
      // after an abort the flag cuts the wait short: drain the MMAs still in
      // flight before tensor memory is freed
      if (!mbar_wait(&bars->done, 0, abort_flag, a.err, kTimeoutNs))
        mbar_drain(&bars->done, 0, 1000000ull);
    }
  } else {
    regs_inc<kRegsSoftmax>();
    // ------------------------------------------------------------- softmax
    const int x = warp >> 2, quad = warp & 3;
    const int row = quad * 32 + lane;
    const int half = row >> 6, iloc = row & 63;
    const int myr = 2 * tile + half;
    const int bh = x ? bhB : bhA;
    const uint32_t tLane = tmem + ((uint32_t)(quad * 32) << 16);
    const uint32_t tS = tLane + kColS, tP = tLane + kColP + x * 64, tO = tLane + kColO + x * 128;
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
      // copy the whole S tile out and hand the buffer to the other tile
      uint32_t v[128];
#pragma unroll
      for (int q = 0; q < 4; ++q) tmem_ld32(tS + q * 32, *reinterpret_cast<uint32_t(*)[32]>(v + q * 32));
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&bars->s_free[x]);
      float smax[2];
#pragma unroll
      for (int s = 0; s < 2; ++s) {
        uint32_t* w = v + s * 64;
        if (kind[s] == kDiag) {
#pragma unroll
          for (int k = 0; k < 64; ++k)
            if (k > iloc) w[k] = __float_as_uint(-INFINITY);
        }
        float a0 = -INFINITY, a1 = -INFINITY, a2 = -INFINITY, a3 = -INFINITY;
#pragma unroll
        for (int k = 0; k < 64; k += 8) {
          a0 = max3(a0, __uint_as_float(w[k]), __uint_as_float(w[k + 1]));
          a1 = max3(a1, __uint_as_float(w[k + 2]), __uint_as_float(w[k + 3]));
          a2 = max3(a2, __uint_as_float(w[k + 4]), __uint_as_float(w[k + 5]));
          a3 = max3(a3, __uint_as_float(w[k + 6]), __uint_as_float(w[k + 7]));
        }
        const float raw = fmaxf(fmaxf(a0, a1), fmaxf(a2, a3));
        smax[s] = kind[s] == kMasked ? -INFINITY : fmaf(raw, sc, bias[s]);
      }
      const float mx = fmaxf(smax[0], smax[1]);
      const bool need = mx > m + kRescaleThreshold;
      if (j > 0) {
        // PV_x(j-1) has read P_x and written O
        if (!mbar_wait(&bars->pv_done[x], (j - 1) & 1, abort_flag, a.err, kTimeoutNs)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (__any_sync(0xffffffffu, need)) {
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
      }
      if (need) m = mx;
      const float mu = m == -INFINITY ? 0.f : m;
      float l0 = 0.f, l1 = 0.f, l2 = 0.f, l3 = 0.f;
      // P of keys [32c, 32c + 32) -> P_x columns [16c, 16c + 16)
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int s = c >> 1;
        uint32_t pk[16];
        if (kind[s] == kMasked) {
#pragma unroll
          for (int k = 0; k < 16; ++k) pk[k] = 0u;
        } else {
          const float cst = bias[s] - mu;
#pragma unroll
          for (int k = 0; k < 32; k += 4) {
            const float p0 = ex2(fmaf(__uint_as_float(v[c * 32 + k]), sc, cst));
            const float p1 = ex2(fmaf(__uint_as_float(v[c * 32 + k + 1]), sc, cst));
            const float p2 = ex2(fmaf(__uint_as_float(v[c * 32 + k + 2]), sc, cst));
            const float p3 = ex2(fmaf(__uint_as_float(v[c * 32 + k + 3]), sc, cst));
            l0 += p0;
            l1 += p1;
            l2 += p2;
            l3 += p3;
            pk[k / 2] = cvt_bf16x2(p0, p1);
            pk[k / 2 + 1] = cvt_bf16x2(p2, p3);
          }
        }
        tmem_st16(tP + c * 16, pk);
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
  // setmaxnreg.inc waits until the registers it asks for are free: launch only
  // if the kernel starts with enough registers per thread for the split
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, kern);
  if (e != cudaSuccess) return e;
  if (fa.numRegs * kThreads < 128 * (2 * kRegsSoftmax + kRegsControl)) return cudaErrorInvalidConfiguration;
  const int smem = Layout2<D>::kSmemBytes;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
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
