// fwd_tq.cu — K2 sparse forward with the keys on the TMEM lanes.
//
// Per CTA: one 64-query block r of one (batch, q-head). Its attended blocks
// (the Top-K list, or threshold list, of K1 plus the current block r) are
// walked two per stage (128 keys). Every computed pair is attended: unlike
// the paired-query-block tiling, no stage carries rows that did not select
// its keys.
//
//   S^T = K_stage . Q^T   M = 128 keys (TMEM lanes), N = 64 queries, K = d
//   O^T += V^T . P^T      M = d = 128 (TMEM lanes), N = 64 queries, K = 128 keys
//
// Softmax statistics run along the TMEM lanes. Row maxima (one per query)
// live in shared memory; each stage exponentiates against them, and a vote of
// the eight softmax warps sends the CTA to a slow path when a logit passes
// its row's maximum by 2^8: exact maxima by warp reductions and a shared-memory
// exchange, rescale of the O^T columns and of the partial row sums. Row sums
// are per-lane partials reduced once at the end.
//
// Warps 0-7 softmax/epilogue (warp w: lane quadrant w%4, query half w/4),
// warp 8 TMA producer, warp 9 TMEM allocator + MMA issuer. TMEM: S^T buffers
// at columns 0 and 64, O^T at 128. Every wait is bounded.
#include <cuda.h>
#include <stdio.h>

#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace gbs {

namespace {

using namespace sm100;

constexpr int kQ = 64;             // queries per CTA
constexpr int kSlot = 64;          // keys per slot (one context block)
constexpr int kBN = 2 * kSlot;     // keys per stage
constexpr int kSoftWarps = 8;
constexpr int kTmaWarp = kSoftWarps, kMmaWarp = kSoftWarps + 1;
constexpr int kThreads = (kSoftWarps + 2) * 32;
constexpr int kSoftThreads = kSoftWarps * 32;
constexpr int kTmemCols = 256;
constexpr uint64_t kTimeoutNs = 4000000000ull;
constexpr float kRescale = 8.0f;   // log2 units
constexpr int D = 128;

struct Layout {
  static constexpr int kChunks = D / 64;
  static constexpr int kQChunk = kQ * 128;     // 8 KB: 64 rows x 128 B
  static constexpr int kKVChunk = kBN * 128;   // 16 KB: 128 rows x 128 B
  static constexpr int kQOff = 0;
  static constexpr int kKOff = kQOff + kChunks * kQChunk;
  static constexpr int kVOff = kKOff + kChunks * kKVChunk;
  static constexpr int kPOff = kVOff + kChunks * kKVChunk;   // P^T: 128 keys x 64 queries bf16
  static constexpr int kRedOff = kPOff + kBN * 128;          // [4 quadrants][64] f32
  static constexpr int kMOff = kRedOff + 4 * kQ * 4;         // [2 epochs][64] f32 row maxima
  static constexpr int kBarOff = kMOff + 2 * kQ * 4;
  static constexpr int kSmemBytes = kBarOff + 256 + 1024;
};
static_assert(Layout::kKOff % 1024 == 0 && Layout::kVOff % 1024 == 0 && Layout::kPOff % 1024 == 0,
              "swizzled tiles need 1024-byte alignment");

struct Bars {
  uint64_t q_full, k_full, v_full, k_empty;
  uint64_t s_full[2];
  uint64_t p_full;  // every softmax thread wrote its P^T row (and any O^T rescale)
  uint64_t p_free;  // PV of the stage finished: P^T and V may be overwritten, O^T is quiescent
  uint64_t vote;    // every softmax thread has voted for the stage
  uint64_t red;     // slow path / epilogue: per-quadrant column values written
  uint64_t mset;    // slow path: next epoch's row maxima written
  uint64_t done;
  uint32_t tmem_base;
  int abort_flag;
  int vote_word[2];
};

struct TqArgs {
  Problem p;
  Selection sel;
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

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Entry e of the CTA's list: the selected blocks in K1's order, then the
// current block (causal, bias 0), then one masked pad (current block again).
__device__ __forceinline__ int entry_block(const TqArgs& a, size_t row, int r, int n_hist, int e) {
  return e < n_hist ? dcheck(__ldg(a.sel.idx + row * a.p.topk + e), 0, r - 1, a.err) : r;
}

__global__ void __launch_bounds__(kThreads, 2)
fwd_tq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
              const __grid_constant__ CUtensorMap tmV, TqArgs a) {
  using L = Layout;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  Bars* bars = reinterpret_cast<Bars*>(smem + L::kBarOff);
  float* red = reinterpret_cast<float*>(smem + L::kRedOff);
  float* m_s = reinterpret_cast<float*>(smem + L::kMOff);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // heavy query blocks first; consecutive CTAs are the heads of one block
  const int BH = a.p.B * a.p.Hq;
  const int r = a.p.Nb - 1 - (int)(blockIdx.x / BH);
  const int bh = (int)(blockIdx.x % BH);
  const int b = bh / a.p.Hq, h = bh % a.p.Hq;
  const int kvz = b * a.p.Hkv + h / a.p.G;
  const size_t row = (size_t)bh * a.p.Nb + r;
  const int n_hist = dcheck(__ldg(a.sel.cnt + row), 0, min(a.p.topk, r), a.err);
  const int n_stages = (n_hist + 2) / 2;  // n_hist + 1 entries, two per stage

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    mbar_init(&bars->k_full, 1);
    mbar_init(&bars->v_full, 1);
    mbar_init(&bars->k_empty, 1);
    mbar_init(&bars->s_full[0], 1);
    mbar_init(&bars->s_full[1], 1);
    mbar_init(&bars->p_full, kSoftThreads);
    mbar_init(&bars->p_free, 1);
    mbar_init(&bars->vote, kSoftThreads);
    mbar_init(&bars->red, kSoftThreads);
    mbar_init(&bars->mset, kSoftThreads);
    mbar_init(&bars->done, 1);
    bars->abort_flag = 0;
    bars->vote_word[0] = 0;
    bars->vote_word[1] = 0;
    fence_barrier_init();
  }
  if (threadIdx.x < 2 * kQ) m_s[threadIdx.x] = -INFINITY;
  if (warp == kTmaWarp && lane == 0) {
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
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

  if (warp == kTmaWarp) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      constexpr uint32_t kSlotBytes = kSlot * 128;
      mbar_arrive_expect_tx(&bars->q_full, L::kChunks * L::kQChunk);
      for (int ch = 0; ch < L::kChunks; ++ch)
        tma_load_3d(smem + L::kQOff + ch * L::kQChunk, &tmQ, &bars->q_full, ch * 64, r * kQ, bh);
      int issued = 0;
      for (int j = 0; j < n_stages; ++j) {
        const int c0 = entry_block(a, row, r, n_hist, 2 * j);
        const int c1 = entry_block(a, row, r, n_hist, 2 * j + 1);
        uint8_t* kst = smem + L::kKOff;
        uint8_t* vst = smem + L::kVOff;
        // K is free once S^T of the previous stage has read it
        if (j > 0 && !mbar_wait(&bars->k_empty, (j - 1) & 1, abort_flag, a.err, kTimeoutNs)) break;
        mbar_arrive_expect_tx(&bars->k_full, L::kChunks * L::kKVChunk);
        for (int ch = 0; ch < L::kChunks; ++ch) {
          tma_load_3d(kst + ch * L::kKVChunk, &tmK, &bars->k_full, ch * 64, c0 * kSlot, kvz);
          tma_load_3d(kst + ch * L::kKVChunk + kSlotBytes, &tmK, &bars->k_full, ch * 64,
                      c1 * kSlot, kvz);
        }
        // V is free once PV of the previous stage has read it
        if (j > 0 && !mbar_wait(&bars->p_free, (j - 1) & 1, abort_flag, a.err, kTimeoutNs)) break;
        mbar_arrive_expect_tx(&bars->v_full, L::kChunks * L::kKVChunk);
        for (int ch = 0; ch < L::kChunks; ++ch) {
          tma_load_3d(vst + ch * L::kKVChunk, &tmV, &bars->v_full, ch * 64, c0 * kSlot, kvz);
          tma_load_3d(vst + ch * L::kKVChunk + kSlotBytes, &tmV, &bars->v_full, ch * 64,
                      c1 * kSlot, kvz);
        }
        issued = j + 1;
      }
      if (*abort_flag) {  // let the loads in flight land before the CTA exits
        mbar_wait(&bars->q_full, 0, abort_flag, nullptr, 1000000ull);
        if (issued > 0) {
          mbar_wait(&bars->k_full, (issued - 1) & 1, abort_flag, nullptr, 1000000ull);
          mbar_wait(&bars->v_full, (issued - 1) & 1, abort_flag, nullptr, 1000000ull);
        }
      }
    }
  } else if (warp == kMmaWarp) {
    // -------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(kBN, kQ, 0, 0);  // S^T: K and Q K-major
      constexpr uint32_t idO = idesc_bf16_f32(D, kQ, 1, 1);    // O^T: V and P^T MN-major
      const uint32_t q_addr = smem_u32(smem + L::kQOff);
      const uint32_t k_addr = smem_u32(smem + L::kKOff), v_addr = smem_u32(smem + L::kVOff);
      const uint32_t p_addr = smem_u32(smem + L::kPOff);
      const uint32_t tO = tmem + 128;
      bool ok = mbar_wait(&bars->q_full, 0, abort_flag, a.err, kTimeoutNs);
      auto issue_s = [&](int j) -> bool {
        if (!mbar_wait(&bars->k_full, j & 1, abort_flag, a.err, kTimeoutNs)) return false;
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const int ch = ks >> 2, kk = ks & 3;
          mma_ss(tmem + (j & 1) * 64, sdesc_sw128(k_addr + ch * L::kKVChunk + kk * 32, 16, 1024),
                 sdesc_sw128(q_addr + ch * L::kQChunk + kk * 32, 16, 1024), idS, ks > 0 ? 1u : 0u);
        }
        mma_commit(&bars->s_full[j & 1]);
        mma_commit(&bars->k_empty);
        return true;
      };
      if (ok) ok = issue_s(0);
      if (ok && n_stages > 1) ok = issue_s(1);
      for (int j = 0; ok && j < n_stages; ++j) {
        // O^T += V_j^T P_j^T once the softmax has written P_j^T
        if (!mbar_wait(&bars->p_full, j & 1, abort_flag, a.err, kTimeoutNs) ||
            !mbar_wait(&bars->v_full, j & 1, abort_flag, a.err, kTimeoutNs))
          break;
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < kBN / 16; ++ks)
          mma_ss(tO, sdesc_sw128(v_addr + ks * 16 * 128, L::kKVChunk, 1024),
                 sdesc_sw128(p_addr + ks * 16 * 128, L::kKVChunk, 1024), idO,
                 (j > 0 || ks > 0) ? 1u : 0u);
        mma_commit(&bars->p_free);
        // S^T of stage j + 2 reuses the buffer stage j's softmax has finished with
        if (j + 2 < n_stages && !issue_s(j + 2)) break;
      }
      mma_commit(&bars->done);
      mbar_wait(&bars->done, 0, abort_flag, a.err, kTimeoutNs);
    }
  } else {
    // ------------------------------------------------- softmax + epilogue
    const int quad = warp & 3, half = warp >> 2;
    const int t = quad * 32 + lane;        // key row of the stage == O^T row (d index)
    const int col0 = half * 32;            // this warp's 32 query columns
    const int slot = t >> 6, kk = t & 63;  // which block of the stage, key within it
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    // partial row sums of this lane's keys live in TMEM columns 192 + col0 + k
    const uint32_t l_addr = tmem + 192 + lane_off + col0;
    const uint32_t o_addr = tmem + 128 + lane_off + col0;
    const float sc = a.p.scale_log2;
    uint8_t* prow = smem + L::kPOff + t * 128;
    {
      uint32_t zero[16];
#pragma unroll
      for (int k = 0; k < 16; ++k) zero[k] = 0u;
      tmem_st16(l_addr, zero);
      tmem_st16(l_addr + 16, zero);
      tmem_wait_st();
    }
    int epoch = 0;
    bool ok = true;
    for (int j = 0; j < n_stages; ++j) {
      const int e = 2 * j + slot;
      int kind = kMasked;
      float bias = 0.f;
      if (e < n_hist) {
        kind = kFull;
        bias = __ldg(a.sel.logg + row * a.p.topk + e) * GBS_LOG2E;
      } else if (e == n_hist) {
        kind = kDiag;
      }
      if (!mbar_wait(&bars->s_full[j & 1], (j >> 1) & 1, abort_flag, a.err, kTimeoutNs)) {
        ok = false;
        break;
      }
      tc_fence_after();
      // 16 of the stage's logits, scaled and biased (log2 units). S^T stays in
      // TMEM until this stage's P^T is handed over, so each phase below reloads
      // it instead of keeping the values live across the barriers.
      const uint32_t s_addr = tmem + (j & 1) * 64 + lane_off + col0;
      auto load_z = [&](int c, float (&z)[16]) {
        uint32_t v[16];
        tmem_ld16(s_addr + c * 16, v);
        tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const bool masked = kind == kMasked || (kind == kDiag && kk > col0 + c * 16 + k);
          z[k] = masked ? -INFINITY : fmaf(__uint_as_float(v[k]), sc, bias);
        }
      };
      // vote: does any logit pass its row's maximum by more than 2^8?
      const float* m_cur = m_s + (epoch & 1) * kQ + col0;
      bool over = false;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        float z[16];
        load_z(c, z);
#pragma unroll
        for (int k = 0; k < 16; k += 4) {
          const float4 m4 = *reinterpret_cast<const float4*>(m_cur + c * 16 + k);
          over |= z[k] > m4.x + kRescale;
          over |= z[k + 1] > m4.y + kRescale;
          over |= z[k + 2] > m4.z + kRescale;
          over |= z[k + 3] > m4.w + kRescale;
        }
      }
      if (__any_sync(0xffffffffu, over) && lane == 0)
        reinterpret_cast<volatile int*>(bars->vote_word)[j & 1] = j + 1;
      mbar_arrive(&bars->vote);
      if (!mbar_wait(&bars->vote, j & 1, abort_flag, a.err, kTimeoutNs)) {
        ok = false;
        break;
      }
      const bool slow = reinterpret_cast<volatile int*>(bars->vote_word)[j & 1] == j + 1;
      // O^T may be rescaled and P^T overwritten only after PV of stage j - 1
      if (j > 0 && !mbar_wait(&bars->p_free, (j - 1) & 1, abort_flag, a.err, kTimeoutNs)) {
        ok = false;
        break;
      }
      if (slow) {
        // exact maxima: per-quadrant column maxima through shared memory
        float mine = -INFINITY;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          float z[16];
          load_z(c, z);
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            const float mx = warp_max(z[k]);
            if (lane == c * 16 + k) mine = mx;
          }
        }
        red[quad * kQ + col0 + lane] = mine;
        mbar_arrive(&bars->red);
        if (!mbar_wait(&bars->red, epoch & 1, abort_flag, a.err, kTimeoutNs)) {
          ok = false;
          break;
        }
        float* m_next = m_s + ((epoch + 1) & 1) * kQ + col0;
        // rescale the partial sums and this lane's O^T row, 16 columns at a time
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t o[16], lv[16];
          tmem_ld16(l_addr + c * 16, lv);
          if (j > 0) tmem_ld16(o_addr + c * 16, o);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            const int q = col0 + c * 16 + k;
            const float mo = m_cur[c * 16 + k];
            const float mn = fmaxf(fmaxf(mo, fmaxf(red[q], red[kQ + q])),
                                   fmaxf(red[2 * kQ + q], red[3 * kQ + q]));
            const float f = mo == -INFINITY ? 0.f : ex2(mo - mn);
            lv[k] = __float_as_uint(__uint_as_float(lv[k]) * f);
            o[k] = __float_as_uint(__uint_as_float(o[k]) * f);
            if (quad == 0 && lane == 0) m_next[c * 16 + k] = mn;
          }
          tmem_st16(l_addr + c * 16, lv);
          if (j > 0) tmem_st16(o_addr + c * 16, o);
        }
        tmem_wait_st();
        mbar_arrive(&bars->mset);
        if (!mbar_wait(&bars->mset, epoch & 1, abort_flag, a.err, kTimeoutNs)) {
          ok = false;
          break;
        }
        ++epoch;
      }
      // P^T row of this key: p = 2^(z - m), partial row sums; 16 query columns
      // (two 16-byte units of the 128-byte swizzled row) at a time
      const float* m_use = m_s + (epoch & 1) * kQ + col0;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        float z[16];
        uint32_t lv[16];
        tmem_ld16(l_addr + c * 16, lv);
        load_z(c, z);  // its wait also covers the partial sums
        uint32_t pk[8];
#pragma unroll
        for (int k = 0; k < 16; k += 4) {
          const float4 m4 = *reinterpret_cast<const float4*>(m_use + c * 16 + k);
          const float p0 = ex2(z[k] - m4.x), p1 = ex2(z[k + 1] - m4.y);
          const float p2 = ex2(z[k + 2] - m4.z), p3 = ex2(z[k + 3] - m4.w);
          lv[k] = __float_as_uint(__uint_as_float(lv[k]) + p0);
          lv[k + 1] = __float_as_uint(__uint_as_float(lv[k + 1]) + p1);
          lv[k + 2] = __float_as_uint(__uint_as_float(lv[k + 2]) + p2);
          lv[k + 3] = __float_as_uint(__uint_as_float(lv[k + 3]) + p3);
          pk[k / 2] = pack_bf16(p0, p1);
          pk[k / 2 + 1] = pack_bf16(p2, p3);
        }
        tmem_st16(l_addr + c * 16, lv);
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int u = half * 4 + c * 2 + i;  // 16-byte unit of the row, 128-byte swizzle
          *reinterpret_cast<uint4*>(prow + ((u ^ (t & 7)) << 4)) =
              make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
        }
      }
      tmem_wait_st();
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&bars->p_full);
    }
    // epilogue: row sums across the 128 key lanes, then O = (O^T)^T / l
    if (ok && mbar_wait(&bars->done, 0, abort_flag, a.err, kTimeoutNs)) {
      tc_fence_after();
      float mine = 0.f;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t lv[16];
        tmem_ld16(l_addr + c * 16, lv);
        tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const float sum = warp_sum(__uint_as_float(lv[k]));
          if (lane == c * 16 + k) mine = sum;
        }
      }
      red[quad * kQ + col0 + lane] = mine;
      mbar_arrive(&bars->red);
      if (mbar_wait(&bars->red, epoch & 1, abort_flag, a.err, kTimeoutNs)) {
        const float* m_fin = m_s + (epoch & 1) * kQ + col0;
        __nv_bfloat16* obase = a.O + ((size_t)bh * a.p.N + (size_t)r * kQ + col0) * D + t;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t o[16];
          tmem_ld16(o_addr + c * 16, o);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            const int q = col0 + c * 16 + k;
            const float lsum = (red[q] + red[kQ + q]) + (red[2 * kQ + q] + red[3 * kQ + q]);
            obase[(size_t)(c * 16 + k) * D] = __float2bfloat16_rn(__uint_as_float(o[k]) / lsum);
            if (quad == 0 && lane == c * 16 + k)
              a.LSE[(size_t)bh * a.p.N + (size_t)r * kQ + q] =
                  (m_fin[c * 16 + k] + log2f(lsum)) * GBS_LN2;
          }
        }
      }
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

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

bool make_map(CUtensorMap* m, const void* base, int d, int rows, int heads, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)rows, (cuuint64_t)heads};
  const cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)d * rows * 2};
  const cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool fwd_tq_supported(const Problem& p) {
  return p.mode != GBS_TRAIN && p.dtype == GBS_BF16 && p.bs == kSlot && p.d == D &&
         p.N % kSlot == 0;
}

cudaError_t launch_fwd_tq(const Problem& p, const void* Q, const void* K, const void* V,
                          const Selection& sel, void* O, float* LSE, unsigned int* err,
                          cudaStream_t st) {
  if (!fwd_tq_supported(p)) return cudaErrorNotSupported;
  TqArgs a;
  a.p = p;
  a.sel = sel;
  a.O = reinterpret_cast<__nv_bfloat16*>(O);
  a.LSE = LSE;
  a.err = err;
  CUtensorMap tq, tk, tv;
  if (!make_map(&tq, Q, D, p.N, p.B * p.Hq, kQ) || !make_map(&tk, K, D, p.N, p.B * p.Hkv, kSlot) ||
      !make_map(&tv, V, D, p.N, p.B * p.Hkv, kSlot))
    return cudaErrorInvalidValue;
  const int smem = Layout::kSmemBytes;
  cudaError_t e =
      cudaFuncSetAttribute(fwd_tq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const unsigned grid = (unsigned)(p.B * p.Hq * p.Nb);
  timer_begin(GBS_OP_FWD, st);
  fwd_tq_kernel<<<grid, kThreads, smem, st>>>(tq, tk, tv, a);
  timer_end(GBS_OP_FWD, st);
  note_launch();
  return cudaGetLastError();
}

}  // namespace gbs
