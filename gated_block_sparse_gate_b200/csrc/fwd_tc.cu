// fwd_tc.cu — K2: gated flash-attention forward on the 5th-generation tensor
// cores (tcgen05, sm_100a), bf16 in, fp32 accumulate.
//
// Computes, per query row i, O_i = softmax_j(z_ij) V and LSE_i with
// z_ij = scale * q_i.k_j + b_ij: b_ij is the normalised log gate of key block
// c(j) for query block r(i) when c(j) is an attended historical block, 0 for
// the current block with j <= i, -inf otherwise (ai.viyan.live, "SAS Learns
// Token Importance for Sparse Attention", "The Logit Injection Mechanism";
// Hugging Face paper page of "SAS: Simple Attention Sparsification via
// End-to-End Optimization of Context Ranking", Abstract). Training mode visits
// every block c <= r; sparse mode visits the Top-K list of K1 plus the current
// block (NeurIPS 2026 poster page, Abstract). Blocks are processed one tile at
// a time with an online softmax; the N x N matrix is never formed (blog,
// "Implementation and Efficiency").
//
// Tiling: one CTA per (batch, q-head, 128-row query tile = two 64-row query
// blocks). Each pipeline stage brings 128 keys = two 64-key "slots"; a slot is
// one context block, so in sparse mode the two slots of a stage can be any two
// blocks of the union of the tile's two selection lists (a per-tile "plan"
// built by plan_kernel). Per slot and per query-block half the softmax applies
// one scalar bias (log gate), a causal mask (current block) or -inf.
//
// Warp roles (192 threads): warps 0-3 softmax/epilogue (thread = query row =
// TMEM lane), warp 4 TMA producer, warp 5 TMEM allocator + MMA issuer.
// Two CTAs share an SM (96 KB of shared memory and 256 TMEM columns each), so
// one CTA's softmax runs while the other's S and PV MMAs do; inside a CTA the
// stages are serial: S_j -> softmax -> PV_j -> S_{j+1}. TMEM: S at column 0
// (128 fp32 columns), O at 128; P is written back as bf16 over the first 64
// columns of S and read by the PV MMA from TMEM. K and V have one stage each:
// the next K loads as soon as S has read the current one, the next V as soon
// as PV has. Measured on the N = 65536 sparse prefill, this runs 25-34%
// faster than two tiles ping-ponging inside one CTA over 64-key slots.
// S = Q K^T: M=128, N=128, K=16 per instruction, both operands K-major,
// 128-byte swizzled tiles loaded by TMA. O += P V: A = P from TMEM, B = V
// MN-major (V rows are keys, contiguous in d).
// The O rescale is lazy: the running max only moves when a row's new max
// exceeds it by more than 2^8, which keeps the result exact (the final
// normalisation uses the same max) while avoiding most TMEM round trips.
// Every mbarrier wait is bounded; on expiry the kernel records
// GBS_ERR_TIMEOUT, drains its MMAs and loads, frees TMEM and returns.
#include <cuda.h>
#include <stdio.h>

#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace gbs {

namespace {

using namespace sm100;

constexpr int kBM = 128;            // query rows per tile
constexpr int kSlot = 64;           // keys per slot (one context block)
constexpr int kBN = 2 * kSlot;      // keys per stage
constexpr int kThreads = 192;
constexpr int kTmemCols = 256;  // two CTAs per SM share the 512 columns
constexpr uint64_t kTimeoutNs = 4000000000ull;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

template <int D>
struct Layout {
  static constexpr int kChunks = D / 64;                   // 64-column (128-byte) chunks
  static constexpr int kQChunk = kBM * 128;                // bytes per Q chunk
  static constexpr int kKVChunk = kBN * 128;               // bytes per K/V chunk of a stage
  static constexpr int kQBytes = kChunks * kQChunk;
  static constexpr int kKVBytes = kChunks * kKVChunk;      // per stage, per tensor
  static constexpr int kQOff = 0;
  static constexpr int kKOff = kQOff + kQBytes;
  static constexpr int kVOff = kKOff + kKVBytes;   // one K and one V stage
  static constexpr int kBarOff = kVOff + kKVBytes;
  static constexpr int kSmemBytes = kBarOff + 256 + 1024;  // + barriers + alignment slack
};

struct Barriers {
  uint64_t q_full;
  uint64_t k_full;
  uint64_t v_full;
  uint64_t k_empty, v_empty;
  uint64_t s_full;
  uint64_t p_full;
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

struct FwdArgs {
  Problem p;
  const float* S;
  const float* slse;
  const int32_t* plan;
  int plan_stride;
  int n_tiles;           // query tiles per head
  __nv_bfloat16* O;
  float* LSE;
  unsigned int* err;
};

enum : int { kMasked = 0, kDiag = 1, kFull = 2 };

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

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Slot `s` (0 or 1) of stage `j`: the key block to load.
__device__ __forceinline__ int slot_block(const FwdArgs& a, const int32_t* plan_tile, int j, int s) {
  if (a.p.mode == GBS_TRAIN) {
    const int c = 2 * j + s;
    return c < a.p.Nb ? c : 0;  // a block past the end (odd Nb) loads block 0, fully masked
  }
  return plan_tile[1 + 2 * j + s];
}

// Bias (log2 units) of slot `s` of stage `j` for query block `myr` of this
// tile's half `half`: +inf marks the causal current block, -inf a masked slot.
__device__ __forceinline__ float slot_bias(const FwdArgs& a, const int32_t* plan_tile, size_t bh,
                                           int j, int s, int half, int myr) {
  if (a.p.mode == GBS_TRAIN) {
    const int c = 2 * j + s;
    if (myr >= a.p.Nb || c > myr) return -INFINITY;
    if (c == myr) return INFINITY;
    const size_t row = bh * a.p.Nb + myr;
    return (__ldg(a.S + row * a.p.Nb + c) - __ldg(a.slse + row)) * GBS_LOG2E;
  }
  return __int_as_float(__ldg(plan_tile + (1 + half) * a.plan_stride + 2 * j + s));
}

template <int D>
__global__ void __launch_bounds__(kThreads, 2)
fwd_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
              const __grid_constant__ CUtensorMap tmV, FwdArgs a) {
  using L = Layout<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  Barriers* bars = reinterpret_cast<Barriers*>(smem + L::kBarOff);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // heavy tiles first: consecutive CTAs are the heads of one tile (KV reuse in L2)
  const int BH = a.p.B * a.p.Hq;
  const int tile = a.n_tiles - 1 - (int)(blockIdx.x / BH);
  const int bh = (int)(blockIdx.x % BH);
  const int b = bh / a.p.Hq, h = bh % a.p.Hq;
  const int kvz = b * a.p.Hkv + h / a.p.G;
  const int32_t* plan_tile =
      a.p.mode == GBS_TRAIN ? nullptr : a.plan + ((size_t)bh * a.n_tiles + tile) * 3 * a.plan_stride;
  const int n_stages = a.p.mode == GBS_TRAIN ? tile + 1 : (__ldg(plan_tile) >> 1);

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    mbar_init(&bars->k_full, 1);
    mbar_init(&bars->v_full, 1);
    mbar_init(&bars->k_empty, 1);
    mbar_init(&bars->v_empty, 1);
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->p_full, 128);
    mbar_init(&bars->drain, 1);
    bars->abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 4 && lane == 0) {
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
  }
  if (warp == 5) {
    tmem_alloc(&bars->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  volatile int* abort_flag = &bars->abort_flag;

  if (warp == 4) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      constexpr uint32_t kSlotBytes = kSlot * 128;
      mbar_arrive_expect_tx(&bars->q_full, L::kQBytes);
      for (int ch = 0; ch < L::kChunks; ++ch)
        tma_load_3d(smem + L::kQOff + ch * L::kQChunk, &tmQ, &bars->q_full, ch * 64, tile * kBM, bh);
      int issued = 0;
      for (int j = 0; j < n_stages; ++j) {
        const int c0 = slot_block(a, plan_tile, j, 0), c1 = slot_block(a, plan_tile, j, 1);
        uint8_t* kst = smem + L::kKOff;
        uint8_t* vst = smem + L::kVOff;
        // K is free once S of the previous stage has read it
        if (j > 0 && !mbar_wait(&bars->k_empty, (j - 1) & 1, abort_flag, a.err, kTimeoutNs)) break;
        mbar_arrive_expect_tx(&bars->k_full, L::kKVBytes);
        for (int ch = 0; ch < L::kChunks; ++ch) {
          tma_load_3d(kst + ch * L::kKVChunk, &tmK, &bars->k_full, ch * 64, c0 * kSlot, kvz);
          tma_load_3d(kst + ch * L::kKVChunk + kSlotBytes, &tmK, &bars->k_full, ch * 64,
                      c1 * kSlot, kvz);
        }
        // V is free once PV of the previous stage has read it
        if (j > 0 && !mbar_wait(&bars->v_empty, (j - 1) & 1, abort_flag, a.err, kTimeoutNs)) break;
        mbar_arrive_expect_tx(&bars->v_full, L::kKVBytes);
        for (int ch = 0; ch < L::kChunks; ++ch) {
          tma_load_3d(vst + ch * L::kKVChunk, &tmV, &bars->v_full, ch * 64, c0 * kSlot, kvz);
          tma_load_3d(vst + ch * L::kKVChunk + kSlotBytes, &tmV, &bars->v_full, ch * 64,
                      c1 * kSlot, kvz);
        }
        issued = j + 1;
      }
      if (*abort_flag) {
        mbar_drain(&bars->q_full, 0, 1000000ull);
        if (issued > 0) {
          mbar_drain(&bars->k_full, (issued - 1) & 1, 1000000ull);
          mbar_drain(&bars->v_full, (issued - 1) & 1, 1000000ull);
        }
      }
    }
  } else if (warp == 5) {
    // -------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(kBM, kBN, 0);
      constexpr uint32_t idO = idesc_bf16_f32(kBM, D, 1);
      const uint32_t q_addr = smem_u32(smem + L::kQOff);
      const uint32_t tS = tmem, tO = tmem + 128;
      const uint32_t k_addr = smem_u32(smem + L::kKOff), v_addr = smem_u32(smem + L::kVOff);
      bool ok = mbar_wait(&bars->q_full, 0, abort_flag, a.err, kTimeoutNs);
      for (int j = 0; ok && j < n_stages; ++j) {
        // S_j = Q K_j^T (after PV_{j-1} has read P_{j-1} from the same columns)
        if (!mbar_wait(&bars->k_full, j & 1, abort_flag, a.err, kTimeoutNs)) break;
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const int ch = ks >> 2, kk = ks & 3;
          mma_ss(tS, sdesc_sw128(q_addr + ch * L::kQChunk + kk * 32, 16, 1024),
                 sdesc_sw128(k_addr + ch * L::kKVChunk + kk * 32, 16, 1024), idS, ks > 0 ? 1u : 0u);
        }
        mma_commit(&bars->s_full);
        mma_commit(&bars->k_empty);
        // O += P_j V_j
        if (!mbar_wait(&bars->p_full, j & 1, abort_flag, a.err, kTimeoutNs) ||
            !mbar_wait(&bars->v_full, j & 1, abort_flag, a.err, kTimeoutNs))
          break;
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < kBN / 16; ++ks)
          mma_ts(tO, tS + ks * 8, sdesc_sw128(v_addr + ks * 16 * 128, L::kKVChunk, 1024), idO,
                 (j > 0 || ks > 0) ? 1u : 0u);
        mma_commit(&bars->v_empty);
      }
      // drain: every MMA issued above has finished once this arrives
      mma_commit(&bars->drain);
      // after an abort the flag cuts the wait short: drain the MMAs still in
      // flight before tensor memory is freed
      if (!mbar_wait(&bars->drain, 0, abort_flag, a.err, kTimeoutNs))
        mbar_drain(&bars->drain, 0, 1000000ull);
    }
  } else {
    // ----------------------------------------------------- softmax + epilogue
    const int row = warp * 32 + lane;  // TMEM lane == query row in the tile
    const int half = row >> 6, iloc = row & 63;
    const int myr = 2 * tile + half;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    const float sc = a.p.scale_log2;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < n_stages; ++j) {
      // per slot: +inf = causal current block, -inf = masked, else the log2 gate
      const float sb0 = slot_bias(a, plan_tile, bh, j, 0, half, myr);
      const float sb1 = slot_bias(a, plan_tile, bh, j, 1, half, myr);
      const int kind[2] = {sb0 == INFINITY ? kDiag : (sb0 == -INFINITY ? kMasked : kFull),
                           sb1 == INFINITY ? kDiag : (sb1 == -INFINITY ? kMasked : kFull)};
      const float bias[2] = {kind[0] == kFull ? sb0 : 0.f, kind[1] == kFull ? sb1 : 0.f};
      if (!mbar_wait(&bars->s_full, j & 1, abort_flag, a.err, kTimeoutNs)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t tS = tmem + lane_off;
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
        const float rawmax = fmaxf(fmaxf(a0, a1), fmaxf(a2, a3));
        smax[s] = kind[s] == kMasked ? -INFINITY : fmaf(rawmax, sc, bias[s]);
        if (s == 1) {
#pragma unroll
          for (int k = 0; k < 64; ++k) v1[k] = v[k];
        }
      }
      const float mx = fmaxf(smax[0], smax[1]);
      const bool need = mx > m + kRescaleThreshold;
      // O is quiescent: the commit that signalled this S covered the previous PV
      if (__any_sync(0xffffffffu, need) && j > 0) {
        const float f = need ? ex2(m - mx) : 1.f;
        const uint32_t tO = tmem + lane_off + 128;
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
            // pass 1 already set the causal mask's -inf in v1
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
      mbar_arrive(&bars->p_full);
    }
    if (ok && mbar_wait(&bars->drain, 0, abort_flag, a.err, kTimeoutNs)) {
      tc_fence_after();
      const int qrow = tile * kBM + row;
      const bool valid = qrow < a.p.N;
      const float inv = 1.f / l;
      const uint32_t tO = tmem + lane_off + 128;
      __nv_bfloat16* orow = a.O + ((size_t)bh * a.p.N + qrow) * D;
#pragma unroll
      for (int q = 0; q < D / 32; ++q) {
        uint32_t o[32];
        tmem_ld32(tO + q * 32, o);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const __nv_bfloat162 pb = __floats2bfloat162_rn(__uint_as_float(o[2 * k]) * inv,
                                                          __uint_as_float(o[2 * k + 1]) * inv);
          pk[k] = *reinterpret_cast<const uint32_t*>(&pb);
        }
        if (valid) {
          uint4* dst = reinterpret_cast<uint4*>(orow + q * 32);
#pragma unroll
          for (int k = 0; k < 4; ++k) dst[k] = make_uint4(pk[4 * k], pk[4 * k + 1], pk[4 * k + 2], pk[4 * k + 3]);
        }
      }
      if (valid) a.LSE[(size_t)bh * a.p.N + qrow] = (m + log2f(l)) * GBS_LN2;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// Per (batch, head, tile): the ascending union of both query blocks' selected
// lists plus their current blocks, padded to an even slot count, with each
// half's bias per slot (log2 units; +inf = causal current block, -inf = not
// attended by that half).
__global__ void plan_kernel(Problem p, Selection sel, int32_t* __restrict__ plan, int stride,
                            int n_tiles) {
  const int id = blockIdx.x * blockDim.x + threadIdx.x;
  const int BH = p.B * p.Hq;
  if (id >= BH * n_tiles) return;
  const int bh = id / n_tiles, t = id % n_tiles;
  int32_t* out = plan + (size_t)id * 3 * stride;
  int32_t* cs = out + 1;
  float* b0 = reinterpret_cast<float*>(out + stride);
  float* b1 = reinterpret_cast<float*>(out + 2 * stride);
  const int r0 = 2 * t, r1 = 2 * t + 1;
  const bool has1 = r1 < p.Nb;
  const size_t row0 = (size_t)bh * p.Nb + r0, row1 = row0 + 1;
  const int n0 = sel.cnt[row0], n1 = has1 ? sel.cnt[row1] : 0;
  const int32_t* i0 = sel.idx + row0 * p.topk;
  const int32_t* i1 = sel.idx + row1 * p.topk;
  const float* g0 = sel.logg + row0 * p.topk;
  const float* g1 = sel.logg + row1 * p.topk;
  int a0 = 0, a1 = 0, n = 0;
  bool d0 = false, d1 = !has1;
  while (true) {
    // next candidate block from each source (INT_MAX when exhausted)
    const int x0 = a0 < n0 ? i0[a0] : 0x7fffffff;
    const int x1 = a1 < n1 ? i1[a1] : 0x7fffffff;
    const int xd0 = d0 ? 0x7fffffff : r0;
    const int xd1 = d1 ? 0x7fffffff : r1;
    const int c = min(min(x0, x1), min(xd0, xd1));
    if (c == 0x7fffffff) break;
    float v0 = -INFINITY, v1 = -INFINITY;
    if (x0 == c) { v0 = g0[a0++] * GBS_LOG2E; }
    if (xd0 == c) { v0 = INFINITY; d0 = true; }
    if (x1 == c) { v1 = g1[a1++] * GBS_LOG2E; }
    if (xd1 == c) { v1 = INFINITY; d1 = true; }
    cs[n] = c;
    b0[n] = v0;
    b1[n] = v1;
    ++n;
  }
  if (n & 1) {  // pad: reload the last block, attended by nobody
    cs[n] = cs[n - 1];
    b0[n] = -INFINITY;
    b1[n] = -INFINITY;
    ++n;
  }
  out[0] = n;
}

// --------------------------------------------------------------- host side

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

// [rows_per_head, d] bf16 per head, heads stacked: dims (d, rows, heads).
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

template <int D>
cudaError_t launch_typed(const FwdArgs& a, const void* Q, const void* K, const void* V,
                         cudaStream_t st) {
  CUtensorMap tq, tk, tv;
  if (!make_map(&tq, Q, D, a.p.N, a.p.B * a.p.Hq, kBM) ||
      !make_map(&tk, K, D, a.p.N, a.p.B * a.p.Hkv, kSlot) ||
      !make_map(&tv, V, D, a.p.N, a.p.B * a.p.Hkv, kSlot))
    return cudaErrorInvalidValue;
  auto kern = fwd_tc_kernel<D>;
  const int smem = Layout<D>::kSmemBytes;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const unsigned grid = (unsigned)(a.p.B * a.p.Hq * a.n_tiles);
  timer_begin(GBS_OP_FWD, st);
  kern<<<grid, kThreads, smem, st>>>(tq, tk, tv, a);
  timer_end(GBS_OP_FWD, st);
  note_launch();
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_plan(const Problem& p, const Selection& sel, int32_t* plan, int plan_stride,
                        int n_tiles, cudaStream_t st) {
  const int n = p.B * p.Hq * n_tiles;
  plan_kernel<<<(n + 127) / 128, 128, 0, st>>>(p, sel, plan, plan_stride, n_tiles);
  note_launch();
  return cudaGetLastError();
}

bool fwd_tc_supported(const Problem& p) {
  return p.dtype == GBS_BF16 && p.bs == kSlot && (p.d == 64 || p.d == 128) && p.N % kSlot == 0;
}

cudaError_t launch_fwd_tc(const Problem& p, const void* Q, const void* K, const void* V,
                          const float* S, const Selection& sel, const int32_t* plan,
                          int plan_stride, void* O, float* LSE, unsigned int* err,
                          cudaStream_t st) {
  if (!fwd_tc_supported(p)) return cudaErrorNotSupported;
  FwdArgs a;
  a.p = p;
  a.S = S;
  a.slse = sel.slse;
  a.plan = plan;
  a.plan_stride = plan_stride;
  a.n_tiles = (p.Nb + 1) / 2;
  a.O = reinterpret_cast<__nv_bfloat16*>(O);
  a.LSE = LSE;
  a.err = err;
  if (p.mode != GBS_TRAIN) {
    const int n = p.B * p.Hq * a.n_tiles;
    plan_kernel<<<(n + 127) / 128, 128, 0, st>>>(p, sel, const_cast<int32_t*>(plan), plan_stride,
                                                 a.n_tiles);
    note_launch();
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (p.d == 64) return launch_typed<64>(a, Q, K, V, st);
  return launch_typed<128>(a, Q, K, V, st);
}

}  // namespace gbs
