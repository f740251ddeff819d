// fwd_sp.cu — K2, sparse mode: gated forward over the Top-K selected context
// blocks plus the current block, two query tiles per CTA in ping-pong on the
// tcgen05 tensor cores (sm_100a).
//
// Sparse mode attends, for query block r, only the fixed budget of K
// historical blocks with the largest selector scores (NeurIPS 2026 poster page
// of "SAS: Simple Attention Sparsification via End-to-End Optimization of
// Context Ranking", Abstract; HF paper page, Abstract: hard Top-K) plus the
// always-retained current block, with the log gates renormalised over the
// selection; z_ij = scale q_i.k_j + log g (ai.viyan.live, "SAS Learns Token
// Importance for Sparse Attention", "The Logit Injection Mechanism").
//
// A 128-row query tile holds two 64-row query blocks; its slot plan (from K1 +
// plan_kernel) is the ascending union of their selections and current blocks,
// each slot carrying one bias per half (log gate, causal current block or
// -inf when that half did not select it). The CTA owns that tile for two
// q-heads of one kv group (A, B); each tile walks its own plan one context
// block (64 keys) per pipeline stage with its own K / V rings, so the tiles
// never wait for each other's selections, while their MMAs interleave:
// PV_A(j), S_A(j+1), PV_B(j), S_B(j+1). The gathered key blocks come from all
// over the history, so their loads are latency-bound: each tile keeps three K
// slots and two V slots in flight, and K and V have their own producer warps
// so a V slot waiting for its PV never holds up the next K load.
// TMEM: S_A (64 columns), S_B (64), O_A (128), O_B (128). P is written back as
// bf16 over the first 32 columns of its S and read by PV from TMEM.
// S = Q K^T: M=128, N=64, K=16 per instruction (K-major, 128-byte swizzle);
// O += P V: A from TMEM, V MN-major.
// Warps: 0-3 softmax A, 4-7 softmax B, 8 Q/K producer, 9 TMEM + MMA issuer,
// 10 V producer.
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
constexpr int kKStages = 3;  // K slots in flight per tile (S needs them first)
constexpr int kVStages = 2;  // V slots in flight per tile
constexpr int kKWarp = 8, kMmaWarp = 9, kVWarp = 10;
constexpr int kThreads = 352;
constexpr int kTmemCols = 512;
constexpr uint64_t kTimeoutNs = 4000000000ull;
constexpr float kRescaleThreshold = 8.0f;
constexpr int kQChunk = 128 * 128;  // 64 columns x 128 rows of bf16
constexpr int kSChunk = 64 * 128;   // 64 columns x 64 rows of bf16

template <int D>
struct LayoutSp {
  static constexpr int kChunks = D / 64;
  static constexpr int kQTile = kChunks * kQChunk;
  static constexpr int kSlotBytes = kChunks * kSChunk;  // one 64-key K or V block
  static constexpr int kQOff = 0;                           // Q_A, Q_B
  static constexpr int kKOff = 2 * kQTile;                           // K rings: [tile][3]
  static constexpr int kVOff = kKOff + 2 * kKStages * kSlotBytes;    // V rings: [tile][2]
  static constexpr int kBarOff = kVOff + 2 * kVStages * kSlotBytes;
  static constexpr int kSmemBytes = kBarOff + 256;
};

struct BarsSp {
  uint64_t q_full;
  uint64_t k_full[2][kKStages], k_empty[2][kKStages];  // [tile][stage]
  uint64_t v_full[2][kVStages], v_empty[2][kVStages];
  uint64_t s_full[2], p_full[2];
  uint64_t done;
  uint32_t tmem_base;
  int abort_flag;
};

struct SpArgs {
  Problem p;
  const int32_t* plan;
  int plan_stride;
  int n_tiles;
  __nv_bfloat16* O;
  float* LSE;
  unsigned int* err;
};

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

// Number of real slots of a plan (the trailing padding slot, attended by
// neither half, is skipped).
__device__ __forceinline__ int plan_slots(const int32_t* pl, int stride) {
  int n = __ldg(pl);
  if (n > 0) {
    const float b0 = __int_as_float(__ldg(pl + stride + n - 1));
    const float b1 = __int_as_float(__ldg(pl + 2 * stride + n - 1));
    if (b0 == -INFINITY && b1 == -INFINITY) --n;
  }
  return n;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
fwd_sp_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
              const __grid_constant__ CUtensorMap tmV, SpArgs a) {
  using L = LayoutSp<D>;
  extern __shared__ __align__(1024) uint8_t smem[];
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0) set_error(a.err, GBS_ERR_UNSUPPORTED);
    return;
  }
  BarsSp* bars = reinterpret_cast<BarsSp*>(smem + L::kBarOff);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Problem& p = a.p;

  const int pairs = p.B * (p.Hq / 2);
  const int tile = (int)(blockIdx.x / pairs);
  const int pr = (int)(blockIdx.x % pairs);
  const int b = pr / (p.Hq / 2), h0 = 2 * (pr % (p.Hq / 2));
  const int bh[2] = {b * p.Hq + h0, b * p.Hq + h0 + 1};
  const int kvz = b * p.Hkv + h0 / p.G;
  const int32_t* plan[2] = {a.plan + ((size_t)bh[0] * a.n_tiles + tile) * 3 * a.plan_stride,
                            a.plan + ((size_t)bh[1] * a.n_tiles + tile) * 3 * a.plan_stride};
  const int n[2] = {plan_slots(plan[0], a.plan_stride), plan_slots(plan[1], a.plan_stride)};
  const int n_max = n[0] > n[1] ? n[0] : n[1];

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int x = 0; x < 2; ++x) {
      for (int s = 0; s < kKStages; ++s) {
        mbar_init(&bars->k_full[x][s], 1);
        mbar_init(&bars->k_empty[x][s], 1);
      }
      for (int s = 0; s < kVStages; ++s) {
        mbar_init(&bars->v_full[x][s], 1);
        mbar_init(&bars->v_empty[x][s], 1);
      }
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&bars->s_full[x], 1);
      mbar_init(&bars->p_full[x], 128);
    }
    mbar_init(&bars->done, 1);
    bars->abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&bars->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  volatile int* abort_flag = &bars->abort_flag;

  if (warp == kKWarp) {
    // ------------------------------------------------- Q and K producer (TMA)
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      mbar_arrive_expect_tx(&bars->q_full, 2 * L::kQTile);
      for (int x = 0; x < 2; ++x)
        for (int ch = 0; ch < L::kChunks; ++ch)
          tma_load_3d(smem + L::kQOff + x * L::kQTile + ch * kQChunk, &tmQ, &bars->q_full, ch * 64,
                      tile * kBM, bh[x]);
      bool ok = true;
      int issued[2] = {0, 0};
      for (int j = 0; ok && j < n_max; ++j) {
        for (int x = 0; ok && x < 2; ++x) {
          if (j >= n[x]) continue;
          const int st = j % kKStages;
          const int c = __ldg(plan[x] + 1 + j);  // overlaps the wait below
          // the slot is free once S of step j - kKStages has read it
          if (j >= kKStages &&
              !mbar_wait(&bars->k_empty[x][st], (j / kKStages - 1) & 1, abort_flag, a.err, kTimeoutNs)) {
            ok = false;
            break;
          }
          uint8_t* ks = smem + L::kKOff + (x * kKStages + st) * L::kSlotBytes;
          mbar_arrive_expect_tx(&bars->k_full[x][st], L::kSlotBytes);
          for (int ch = 0; ch < L::kChunks; ++ch)
            tma_load_3d(ks + ch * kSChunk, &tmK, &bars->k_full[x][st], ch * 64, c * kSlot, kvz);
          issued[x] = j + 1;
        }
      }
      if (*abort_flag) {  // let loads still in flight land before the CTA exits
        mbar_wait(&bars->q_full, 0, abort_flag, nullptr, 1000000ull);
        for (int x = 0; x < 2; ++x)
          for (int j = issued[x] - kKStages < 0 ? 0 : issued[x] - kKStages; j < issued[x]; ++j)
            mbar_wait(&bars->k_full[x][j % kKStages], (j / kKStages) & 1, abort_flag, nullptr,
                      1000000ull);
      }
    }
  } else if (warp == kVWarp) {
    // ------------------------------------------------------ V producer (TMA)
    if (lane == 0) {
      prefetch_tmap(&tmV);
      bool ok = true;
      int issued[2] = {0, 0};
      for (int j = 0; ok && j < n_max; ++j) {
        for (int x = 0; ok && x < 2; ++x) {
          if (j >= n[x]) continue;
          const int st = j % kVStages;
          const int c = __ldg(plan[x] + 1 + j);
          // the slot is free once PV of step j - kVStages has read it
          if (j >= kVStages &&
              !mbar_wait(&bars->v_empty[x][st], (j / kVStages - 1) & 1, abort_flag, a.err, kTimeoutNs)) {
            ok = false;
            break;
          }
          uint8_t* vs = smem + L::kVOff + (x * kVStages + st) * L::kSlotBytes;
          mbar_arrive_expect_tx(&bars->v_full[x][st], L::kSlotBytes);
          for (int ch = 0; ch < L::kChunks; ++ch)
            tma_load_3d(vs + ch * kSChunk, &tmV, &bars->v_full[x][st], ch * 64, c * kSlot, kvz);
          issued[x] = j + 1;
        }
      }
      if (*abort_flag) {
        for (int x = 0; x < 2; ++x)
          for (int j = issued[x] - kVStages < 0 ? 0 : issued[x] - kVStages; j < issued[x]; ++j)
            mbar_wait(&bars->v_full[x][j % kVStages], (j / kVStages) & 1, abort_flag, nullptr,
                      1000000ull);
      }
    }
  } else if (warp == kMmaWarp) {
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(kBM, kSlot, 0);
      constexpr uint32_t idO = idesc_bf16_f32(kBM, D, 1);
      auto issue_s = [&](int x, int j) -> bool {
        const int st = j % kKStages;
        if (!mbar_wait(&bars->k_full[x][st], (j / kKStages) & 1, abort_flag, a.err, kTimeoutNs))
          return false;
        tc_fence_after();
        const uint32_t q_addr = smem_u32(smem + L::kQOff + x * L::kQTile);
        const uint32_t k_addr = smem_u32(smem + L::kKOff + (x * kKStages + st) * L::kSlotBytes);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const int ch = ks >> 2, kk = ks & 3;
          mma_ss(tmem + x * 64, sdesc_sw128(q_addr + ch * kQChunk + kk * 32, 16, 1024),
                 sdesc_sw128(k_addr + ch * kSChunk + kk * 32, 16, 1024), idS, ks > 0 ? 1u : 0u);
        }
        mma_commit(&bars->s_full[x]);
        mma_commit(&bars->k_empty[x][st]);
        return true;
      };
      auto issue_pv = [&](int x, int j) -> bool {
        const int st = j % kVStages;
        if (!mbar_wait(&bars->p_full[x], j & 1, abort_flag, a.err, kTimeoutNs)) return false;
        if (!mbar_wait(&bars->v_full[x][st], (j / kVStages) & 1, abort_flag, a.err, kTimeoutNs))
          return false;
        tc_fence_after();
        const uint32_t v_addr = smem_u32(smem + L::kVOff + (x * kVStages + st) * L::kSlotBytes);
#pragma unroll
        for (int ks = 0; ks < kSlot / 16; ++ks)
          mma_ts(tmem + 128 + x * 128, tmem + x * 64 + ks * 8,
                 sdesc_sw128(v_addr + ks * 2048, kSChunk, 1024), idO, (j > 0 || ks > 0) ? 1u : 0u);
        mma_commit(&bars->v_empty[x][st]);
        return true;
      };
      bool ok = mbar_wait(&bars->q_full, 0, abort_flag, a.err, kTimeoutNs);
      tc_fence_after();
      if (ok) ok = issue_s(0, 0);
      if (ok) ok = issue_s(1, 0);
      for (int j = 0; ok && j < n_max; ++j) {
        for (int x = 0; ok && x < 2; ++x) {
          if (j >= n[x]) continue;
          ok = issue_pv(x, j);
          if (ok && j + 1 < n[x]) ok = issue_s(x, j + 1);
        }
      }
      mma_commit(&bars->done);
      mbar_wait(&bars->done, 0, abort_flag, a.err, kTimeoutNs);
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------- softmax
    const int x = warp >> 2, quad = warp & 3;
    const int row = quad * 32 + lane;
    const int half = row >> 6, iloc = row & 63;
    const int32_t* bias_row = plan[x] + (1 + half) * a.plan_stride;
    const uint32_t tS = tmem + ((uint32_t)(quad * 32) << 16) + x * 64;
    const uint32_t tO = tmem + ((uint32_t)(quad * 32) << 16) + 128 + x * 128;
    const float sc = p.scale_log2;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < n[x]; ++j) {
      // +inf: causal current block; -inf: this half did not select the block
      const float bias = __int_as_float(__ldg(bias_row + j));
      if (!mbar_wait(&bars->s_full[x], j & 1, abort_flag, a.err, kTimeoutNs)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t pk[32];
      if (bias == -INFINITY) {
#pragma unroll
        for (int k = 0; k < 32; ++k) pk[k] = 0u;
      } else {
        uint32_t v[64];
        tmem_ld32(tS, *reinterpret_cast<uint32_t(*)[32]>(v));
        tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(v + 32));
        tmem_wait_ld();
        const bool diag = bias == INFINITY;
        if (diag) {
#pragma unroll
          for (int k = 0; k < 64; ++k)
            if (k > iloc) v[k] = __float_as_uint(-INFINITY);
        }
        const float b2 = diag ? 0.f : bias;
        float a0 = -INFINITY, a1 = -INFINITY, a2 = -INFINITY, a3 = -INFINITY;
#pragma unroll
        for (int k = 0; k < 64; k += 8) {
          a0 = max3(a0, __uint_as_float(v[k]), __uint_as_float(v[k + 1]));
          a1 = max3(a1, __uint_as_float(v[k + 2]), __uint_as_float(v[k + 3]));
          a2 = max3(a2, __uint_as_float(v[k + 4]), __uint_as_float(v[k + 5]));
          a3 = max3(a3, __uint_as_float(v[k + 6]), __uint_as_float(v[k + 7]));
        }
        const float mx = fmaf(fmaxf(fmaxf(a0, a1), fmaxf(a2, a3)), sc, b2);
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
        const float cst = b2 - mu;
        float l0 = 0.f, l1 = 0.f, l2 = 0.f, l3 = 0.f;
#pragma unroll
        for (int k = 0; k < 64; k += 4) {
          const float p0 = ex2(fmaf(__uint_as_float(v[k]), sc, cst));
          const float p1 = ex2(fmaf(__uint_as_float(v[k + 1]), sc, cst));
          const float p2 = ex2(fmaf(__uint_as_float(v[k + 2]), sc, cst));
          const float p3 = ex2(fmaf(__uint_as_float(v[k + 3]), sc, cst));
          l0 += p0;
          l1 += p1;
          l2 += p2;
          l3 += p3;
          pk[k / 2] = cvt_bf16x2(p0, p1);
          pk[k / 2 + 1] = cvt_bf16x2(p2, p3);
        }
        l += (l0 + l1) + (l2 + l3);
      }
      tmem_st32(tS, pk);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bars->p_full[x]);
    }
    if (ok && mbar_wait(&bars->done, 0, abort_flag, a.err, kTimeoutNs)) {
      tc_fence_after();
      const int qrow = tile * kBM + row;
      const bool valid = qrow < p.N;
      const float inv = 1.f / l;
      __nv_bfloat16* orow = a.O + ((size_t)bh[x] * p.N + qrow) * D;
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
      if (valid) a.LSE[(size_t)bh[x] * p.N + qrow] = (m + log2f(l)) * GBS_LN2;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

bool make_map_sp(CUtensorMap* m, const void* base, int d, int rows, int heads, int box_rows) {
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
cudaError_t launch_sp(const SpArgs& a, const void* Q, const void* K, const void* V, cudaStream_t st) {
  const Problem& p = a.p;
  CUtensorMap tq, tk, tv;
  if (!make_map_sp(&tq, Q, D, p.N, p.B * p.Hq, kBM) || !make_map_sp(&tk, K, D, p.N, p.B * p.Hkv, kSlot) ||
      !make_map_sp(&tv, V, D, p.N, p.B * p.Hkv, kSlot))
    return cudaErrorInvalidValue;
  auto kern = fwd_sp_kernel<D>;
  const int smem = LayoutSp<D>::kSmemBytes;
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

bool fwd_sp_supported(const Problem& p) {
  return p.dtype == GBS_BF16 && p.mode != GBS_TRAIN && p.bs == kSlot &&
         (p.d == 64 || p.d == 128) && p.N % kSlot == 0 && p.G % 2 == 0;
}

cudaError_t launch_fwd_sp(const Problem& p, const void* Q, const void* K, const void* V,
                          const Selection& sel, int32_t* plan, int plan_stride, void* O,
                          float* LSE, unsigned int* err, cudaStream_t st) {
  if (!fwd_sp_supported(p)) return cudaErrorNotSupported;
  SpArgs a;
  a.p = p;
  a.plan = plan;
  a.plan_stride = plan_stride;
  a.n_tiles = (p.Nb + 1) / 2;
  a.O = reinterpret_cast<__nv_bfloat16*>(O);
  a.LSE = LSE;
  a.err = err;
  cudaError_t e = launch_plan(p, sel, plan, plan_stride, a.n_tiles, st);
  if (e != cudaSuccess) return e;
  if (p.d == 64) return launch_sp<64>(a, Q, K, V, st);
  return launch_sp<128>(a, Q, K, V, st);
}

}  // namespace gbs
