// bwd_kb.cu — K3 sparse backward, one key block per CTA.
//
// CTA = (batch, kv head, 64-key block c). It walks the (q-head, query block r)
// entries of its kv group whose kept set contains c (or r == c), two per step
// (query rows 0-63 and 64-127), so every row of a step attends the step's
// keys. Per step, all products at M = 128:
//   S  = Q K^T,  dP = dO V^T      M = 128 queries (TMEM lanes), N = 64 keys
//   dV^T += dO^T P, dK^T += Q^T dS  M = d = 128 (TMEM lanes), N = 64 keys
//   dQ = dS K                       M = 128 queries, N = d
// P and dS (= dZ, the gradient of the logits) are written once to shared memory
// as bf16 rows (the B operand of dV^T / dK^T, the A operand of dQ). dQ is added
// into the fp32 accumulator by four drain warps. G[r, c] (tile sums of dS) is
// accumulated per warp. Pre/post passes (D = rowsum(dO o O), dQ conversion, dS
// from G) are the training backward's.
//
// Warps: 0-7 compute (lane quadrant w%4 = query rows, key half w/4), 8 TMA,
// 9 TMEM allocator + MMA issuer, 10-13 dQ drain. TMEM (512 columns): S 0,
// dP 64, dV^T 128, dK^T 192, dQ 256. Every wait is bounded.
#include <cuda.h>

#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace gbs {

namespace {

using namespace sm100;

constexpr int D = 128;
constexpr int kBlk = 64;            // keys per CTA, queries per entry
constexpr int kRows = 2 * kBlk;     // query rows per step
constexpr int kComputeWarps = 8;
constexpr int kDrainWarps = 4;
constexpr int kTmaWarp = kComputeWarps, kMmaWarp = kComputeWarps + 1;
constexpr int kThreads = (kComputeWarps + 2 + kDrainWarps) * 32;
constexpr int kTmemCols = 512;
constexpr uint64_t kTimeoutNs = 4000000000ull;

struct Layout {
  static constexpr int kChunks = D / 64;
  static constexpr int kKVChunk = kBlk * 128;    // 8 KB: 64 rows x 128 B
  static constexpr int kQChunk = kRows * 128;    // 16 KB: 128 rows x 128 B
  static constexpr int kKOff = 0;
  static constexpr int kVOff = kKOff + kChunks * kKVChunk;
  static constexpr int kQOff = kVOff + kChunks * kKVChunk;       // 2 stages
  static constexpr int kdOOff = kQOff + 2 * kChunks * kQChunk;   // 2 stages
  static constexpr int kPOff = kdOOff + 2 * kChunks * kQChunk;   // 128 rows x 64 keys bf16
  static constexpr int kSOff = kPOff + kRows * 128;              // dS, same shape
  static constexpr int kBarOff = kSOff + kRows * 128;
  static constexpr int kSmemBytes = kBarOff + 256 + 1024;
  static constexpr int kStage = kChunks * kQChunk;
};
static_assert(Layout::kSmemBytes <= 227 * 1024, "shared memory");

struct Bars {
  uint64_t kv_full;
  uint64_t q_full[2];
  uint64_t stage_free[2];
  uint64_t s_full;    // S and dP of the step in TMEM
  uint64_t ds_full;   // every compute thread wrote its P and dS row
  uint64_t ds_free;   // the step's MMAs have read P and dS
  uint64_t dq_full;   // dQ of the step in TMEM
  uint64_t dq_free;   // the drain warps have read dQ
  uint64_t done;
  uint32_t tmem_base;
  int abort_flag;
};

struct KbArgs {
  Problem p;
  const float* S;
  const float* slse;    // normaliser of the kept set, per (bh, r)
  const float* LSE;
  const float* Dvec;
  float* dQacc;
  float* Gblk;
  __nv_bfloat16* dK;
  __nv_bfloat16* dV;
  const int32_t* plan;  // per CTA: count, then (q-head in group << 16 | r)
  int plan_stride;
  unsigned int* err;
};

enum : int { kMasked = 0, kCausal = 1, kFull = 2 };

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

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Entries of CTA (key block c, batch x kv-head bk): every (q-head, r >= c) of
// the group whose kept bitmap has c, or r == c. One warp per CTA.
__global__ void kb_plan_kernel(const uint32_t* __restrict__ mbits, int mwords, int Nb, int G, int Hq,
                               int Hkv, int BKV, int32_t* __restrict__ plan, int plan_stride) {
  const int lane = threadIdx.x & 31;
  const int id = (int)(blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5));
  if (id >= Nb * BKV) return;
  const int c = id / BKV, bk = id % BKV;
  const int b = bk / Hkv, kvh = bk % Hkv;
  int32_t* out = plan + (size_t)id * plan_stride;
  const int cw = c >> 5, sh = c & 31;
  const uint32_t below = (1u << lane) - 1u;
  int n = 0;
  for (int hh = 0; hh < G; ++hh) {
    const size_t rowbase = (size_t)(b * Hq + kvh * G + hh) * Nb;
    for (int r0 = c; r0 < Nb; r0 += 32) {
      const int r = r0 + lane;
      bool need = false;
      if (r < Nb) need = r == c || ((__ldg(mbits + (rowbase + r) * mwords + cw) >> sh) & 1u);
      const uint32_t m = __ballot_sync(0xffffffffu, need);
      if (need) out[1 + n + __popc(m & below)] = (hh << 16) | r;
      n += __popc(m);
    }
  }
  if (lane == 0) out[0] = n;
}

__global__ void __launch_bounds__(kThreads, 1)
bwd_kb_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
              const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
              KbArgs a) {
  using L = Layout;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  Bars* bars = reinterpret_cast<Bars*>(smem + L::kBarOff);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Problem& p = a.p;

  const int BKV = p.B * p.Hkv;
  const int c = (int)(blockIdx.x / BKV);  // key block; small c = most rows, launched first
  const int bk = (int)(blockIdx.x % BKV);
  const int b = bk / p.Hkv, kvh = bk % p.Hkv;
  const int32_t* list = a.plan + (size_t)blockIdx.x * a.plan_stride;
  const int n_entries = dcheck(__ldg(list), 0, p.G * (p.Nb - c), a.err);
  const int n_steps = (n_entries + 1) >> 1;
  // (batch x q-head row, query block) of entry i; r = -1 past the end
  auto entry_at = [&](int i, int& bh, int& r) {
    int hh = 0;
    r = -1;
    if (i < n_entries) {
      const int e = __ldg(list + 1 + i);
      hh = dcheck(e >> 16, 0, p.G - 1, a.err);
      r = dcheck(e & 0xffff, c, p.Nb - 1, a.err);
    }
    bh = b * p.Hq + kvh * p.G + hh;
  };

  if (threadIdx.x == 0) {
    mbar_init(&bars->kv_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars->q_full[s], 1);
      mbar_init(&bars->stage_free[s], 1);
    }
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->ds_full, kComputeWarps * 32);
    mbar_init(&bars->ds_free, 1);
    mbar_init(&bars->dq_full, 1);
    mbar_init(&bars->dq_free, kDrainWarps * 32);
    mbar_init(&bars->done, 1);
    bars->abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kTmaWarp && lane == 0) {
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
    prefetch_tmap(&tmdO);
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
      const int kvz = b * p.Hkv + kvh;
      mbar_arrive_expect_tx(&bars->kv_full, 2 * L::kChunks * L::kKVChunk);
      for (int ch = 0; ch < L::kChunks; ++ch) {
        tma_load_3d(smem + L::kKOff + ch * L::kKVChunk, &tmK, &bars->kv_full, ch * 64, c * kBlk, kvz);
        tma_load_3d(smem + L::kVOff + ch * L::kKVChunk, &tmV, &bars->kv_full, ch * 64, c * kBlk, kvz);
      }
      int issued = 0;
      for (int j = 0; j < n_steps; ++j) {
        const int st = j & 1;
        // the stage is free once dV^T and dK^T of step j - 2 have read it
        if (j >= 2 &&
            !mbar_wait(&bars->stage_free[st], ((j >> 1) - 1) & 1, abort_flag, a.err, kTimeoutNs))
          break;
        mbar_arrive_expect_tx(&bars->q_full[st], 2 * L::kStage);
        for (int half = 0; half < 2; ++half) {
          int bh, r;
          entry_at(2 * j + half, bh, r);
          if (r < 0) entry_at(2 * j, bh, r);  // a missing second entry reloads the first (masked)
          for (int ch = 0; ch < L::kChunks; ++ch) {
            const int off = st * L::kStage + ch * L::kQChunk + half * kBlk * 128;
            tma_load_3d(smem + L::kQOff + off, &tmQ, &bars->q_full[st], ch * 64, r * kBlk, bh);
            tma_load_3d(smem + L::kdOOff + off, &tmdO, &bars->q_full[st], ch * 64, r * kBlk, bh);
          }
        }
        issued = j + 1;
      }
      if (*abort_flag) {
        mbar_wait(&bars->kv_full, 0, abort_flag, nullptr, 1000000ull);
        for (int j = issued > 2 ? issued - 2 : 0; j < issued; ++j)
          mbar_wait(&bars->q_full[j & 1], (j >> 1) & 1, abort_flag, nullptr, 1000000ull);
      }
    }
  } else if (warp == kMmaWarp) {
    // -------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(kRows, kBlk, 0, 0);  // S, dP: both K-major
      constexpr uint32_t idKV = idesc_bf16_f32(D, kBlk, 1, 1);     // dV^T, dK^T: A, B MN-major
      constexpr uint32_t idQ = idesc_bf16_f32(kRows, D, 1, 0);     // dQ: A = dS K-major, B = K MN-major
      const uint32_t k_addr = smem_u32(smem + L::kKOff), v_addr = smem_u32(smem + L::kVOff);
      const uint32_t p_addr = smem_u32(smem + L::kPOff), ds_addr = smem_u32(smem + L::kSOff);
      const uint32_t tS = tmem, tdP = tmem + 64, tdV = tmem + 128, tdK = tmem + 192,
                     tdQ = tmem + 256;
      bool ok = mbar_wait(&bars->kv_full, 0, abort_flag, a.err, kTimeoutNs);
      auto issue_s = [&](int j) -> bool {
        const int st = j & 1;
        if (!mbar_wait(&bars->q_full[st], (j >> 1) & 1, abort_flag, a.err, kTimeoutNs)) return false;
        tc_fence_after();
        const uint32_t q_addr = smem_u32(smem + L::kQOff + st * L::kStage);
        const uint32_t do_addr = smem_u32(smem + L::kdOOff + st * L::kStage);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const int ch = ks >> 2, kk = ks & 3;
          mma_ss(tS, sdesc_sw128(q_addr + ch * L::kQChunk + kk * 32, 16, 1024),
                 sdesc_sw128(k_addr + ch * L::kKVChunk + kk * 32, 16, 1024), idS, ks > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const int ch = ks >> 2, kk = ks & 3;
          mma_ss(tdP, sdesc_sw128(do_addr + ch * L::kQChunk + kk * 32, 16, 1024),
                 sdesc_sw128(v_addr + ch * L::kKVChunk + kk * 32, 16, 1024), idS, ks > 0 ? 1u : 0u);
        }
        mma_commit(&bars->s_full);
        return true;
      };
      if (ok && n_steps > 0) ok = issue_s(0);
      for (int j = 0; ok && j < n_steps; ++j) {
        const int st = j & 1;
        if (!mbar_wait(&bars->ds_full, j & 1, abort_flag, a.err, kTimeoutNs)) break;
        tc_fence_after();
        const uint32_t q_addr = smem_u32(smem + L::kQOff + st * L::kStage);
        const uint32_t do_addr = smem_u32(smem + L::kdOOff + st * L::kStage);
        // dV^T += dO^T P and dK^T += Q^T dS: K = the step's 128 queries, 16 at a time
#pragma unroll
        for (int ks = 0; ks < kRows / 16; ++ks) {
          mma_ss(tdV, sdesc_sw128(do_addr + ks * 2048, L::kQChunk, 1024),
                 sdesc_sw128(p_addr + ks * 2048, L::kQChunk, 1024), idKV, (j > 0 || ks > 0) ? 1u : 0u);
          mma_ss(tdK, sdesc_sw128(q_addr + ks * 2048, L::kQChunk, 1024),
                 sdesc_sw128(ds_addr + ks * 2048, L::kQChunk, 1024), idKV, (j > 0 || ks > 0) ? 1u : 0u);
        }
        mma_commit(&bars->stage_free[st]);
        // dQ = dS K once the drain warps have emptied the previous step's dQ
        if (j > 0 && !mbar_wait(&bars->dq_free, (j - 1) & 1, abort_flag, a.err, kTimeoutNs)) break;
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < kBlk / 16; ++ks)
          mma_ss(tdQ, sdesc_sw128(ds_addr + ks * 32, 16, 1024),
                 sdesc_sw128(k_addr + ks * 2048, L::kKVChunk, 1024), idQ, ks > 0 ? 1u : 0u);
        mma_commit(&bars->dq_full);
        mma_commit(&bars->ds_free);
        // S and dP of the next step: their TMEM columns were read before ds_full
        if (j + 1 < n_steps && !issue_s(j + 1)) break;
      }
      mma_commit(&bars->done);
      mbar_wait(&bars->done, 0, abort_flag, a.err, kTimeoutNs);
    }
  } else if (warp < kComputeWarps) {
    // ------------------------------------------------------- compute warps
    const int quad = warp & 3, half = warp >> 2;
    const int t = quad * 32 + lane;       // query row of the step == TMEM lane
    const int k0 = half * 32;             // this warp's 32 keys of the block
    const int ent = t >> 6, iloc = t & 63;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const float sc = p.scale_log2;
    uint8_t* prow = smem + L::kPOff + t * 128;
    uint8_t* srow = smem + L::kSOff + t * 128;
    bool ok = true;
    for (int j = 0; j < n_steps; ++j) {
      int bh, r;
      entry_at(2 * j + ent, bh, r);
      int kind = kMasked;
      float bias = 0.f, lse2 = 0.f, dv = 0.f;
      if (r >= 0) {
        const size_t qi = (size_t)bh * p.N + (size_t)r * kBlk + iloc;
        lse2 = __ldg(a.LSE + qi) * GBS_LOG2E;
        dv = __ldg(a.Dvec + qi);
        if (r == c) {
          kind = kCausal;
        } else {
          kind = kFull;
          const size_t row = (size_t)bh * p.Nb + r;
          bias = (__ldg(a.S + row * p.Nb + c) - __ldg(a.slse + row)) * GBS_LOG2E;
        }
      }
      if (!mbar_wait(&bars->s_full, j & 1, abort_flag, a.err, kTimeoutNs) ||
          (j > 0 && !mbar_wait(&bars->ds_free, (j - 1) & 1, abort_flag, a.err, kTimeoutNs))) {
        ok = false;
        break;
      }
      tc_fence_after();
      float g = 0.f;  // sum of dS over this thread's row and keys
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        uint32_t sv[16], pv[16];
        tmem_ld16(tmem + lane_off + k0 + cc * 16, sv);
        tmem_ld16(tmem + 64 + lane_off + k0 + cc * 16, pv);
        tmem_wait_ld();
        uint32_t pp[8], dd[8];
#pragma unroll
        for (int k = 0; k < 16; k += 2) {
          float pr[2], ds[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int key = k0 + cc * 16 + k + e;
            const bool masked = kind == kMasked || (kind == kCausal && key > iloc);
            pr[e] = masked ? 0.f : ex2(fmaf(__uint_as_float(sv[k + e]), sc, bias - lse2));
            ds[e] = pr[e] * (__uint_as_float(pv[k + e]) - dv);
            g += ds[e];
          }
          pp[k / 2] = pack_bf16(pr[0], pr[1]);
          dd[k / 2] = pack_bf16(ds[0], ds[1]);
        }
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int u = half * 4 + cc * 2 + i;  // 16-byte unit of the 128-byte row, swizzled
          *reinterpret_cast<uint4*>(prow + ((u ^ (t & 7)) << 4)) =
              make_uint4(pp[4 * i], pp[4 * i + 1], pp[4 * i + 2], pp[4 * i + 3]);
          *reinterpret_cast<uint4*>(srow + ((u ^ (t & 7)) << 4)) =
              make_uint4(dd[4 * i], dd[4 * i + 1], dd[4 * i + 2], dd[4 * i + 3]);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&bars->ds_full);
      g = warp_sum(g);  // the warp's 32 rows all belong to entry `ent`
      if (lane == 0 && kind != kMasked) atomicAdd(a.Gblk + ((size_t)bh * p.Nb + r) * p.Nb + c, g);
    }
    // epilogue: dV and dK of the block (TMEM lane == d index, column == key)
    if (ok && mbar_wait(&bars->done, 0, abort_flag, a.err, kTimeoutNs)) {
      tc_fence_after();
      const size_t kvrow = ((size_t)(b * p.Hkv + kvh) * p.N + (size_t)c * kBlk + k0) * D + t;
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        __nv_bfloat16* dst = (which == 0 ? a.dV : a.dK) + kvrow;
        const float f = which == 0 ? 1.f : p.scale;
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          uint32_t v[16];
          tmem_ld16(tmem + 128 + which * 64 + lane_off + k0 + cc * 16, v);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 16; ++k)
            dst[(size_t)(cc * 16 + k) * D] = __float2bfloat16_rn(__uint_as_float(v[k]) * f);
        }
      }
    }
  } else {
    // ---------------------------------------------------------- dQ drain warps
    const int quad = warp & 3;  // a warp reaches TMEM lanes 32 * (warp % 4) .. + 31
    const int t = quad * 32 + lane;
    const int ent = t >> 6, iloc = t & 63;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    for (int j = 0; j < n_steps; ++j) {
      int bh, r;
      entry_at(2 * j + ent, bh, r);
      if (!mbar_wait(&bars->dq_full, j & 1, abort_flag, a.err, kTimeoutNs)) break;
      tc_fence_after();
      // a padded second entry (r < 0) reads its TMEM columns but adds nothing
      float* dst = a.dQacc + ((size_t)bh * p.N + (size_t)(r < 0 ? 0 : r) * kBlk + iloc) * D;
#pragma unroll
      for (int cc = 0; cc < D / 16; ++cc) {
        uint32_t v[16];
        tmem_ld16(tmem + 256 + lane_off + cc * 16, v);
        tmem_wait_ld();
        if (r >= 0) {
#pragma unroll
          for (int k = 0; k < 16; k += 4)
            red_add_v4(dst + cc * 16 + k, __uint_as_float(v[k]), __uint_as_float(v[k + 1]),
                       __uint_as_float(v[k + 2]), __uint_as_float(v[k + 3]));
        }
      }
      tc_fence_before();
      mbar_arrive(&bars->dq_free);
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

bool make_map(CUtensorMap* m, const void* base, int d, int rows, int heads) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)rows, (cuuint64_t)heads};
  const cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)d * rows * 2};
  const cuuint32_t box[3] = {64, (cuuint32_t)kBlk, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

size_t bwd_kb_plan_ints(const Problem& p) {
  return (size_t)p.B * p.Hkv * p.Nb * (1 + (size_t)p.G * p.Nb);
}

bool bwd_kb_supported(const Problem& p) {
  return p.mode != GBS_TRAIN && p.dtype == GBS_BF16 && p.bs == kBlk && p.d == D &&
         p.N % kBlk == 0 && p.Nb <= 65536;
}

// The main kernel of the sparse backward. D (Dvec), the zeroed dQ accumulator
// and G, the normaliser slse over the kept set and the kept bitmap come from
// the caller, as for the training backward; dQ conversion and dS follow it.
cudaError_t launch_bwd_kb(const Problem& p, const void* Q, const void* K, const void* V,
                          const float* S, const float* slse, const float* LSE, const void* dO,
                          void* dK, void* dV, const float* Dvec, float* Gblk, float* dQacc,
                          const uint32_t* mbits, int mwords, int32_t* plan, unsigned int* err,
                          cudaStream_t st) {
  if (!bwd_kb_supported(p)) return cudaErrorNotSupported;
  const int BKV = p.B * p.Hkv;
  const int plan_stride = 1 + p.G * p.Nb;
  const int n_ctas = p.Nb * BKV;
  kb_plan_kernel<<<(n_ctas + 3) / 4, 128, 0, st>>>(mbits, mwords, p.Nb, p.G, p.Hq, p.Hkv, BKV, plan,
                                                   plan_stride);
  note_launch();
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  CUtensorMap tq, tk, tv, tdo;
  if (!make_map(&tq, Q, D, p.N, p.B * p.Hq) || !make_map(&tk, K, D, p.N, BKV) ||
      !make_map(&tv, V, D, p.N, BKV) || !make_map(&tdo, dO, D, p.N, p.B * p.Hq))
    return cudaErrorInvalidValue;
  KbArgs a;
  a.p = p;
  a.S = S;
  a.slse = slse;
  a.LSE = LSE;
  a.Dvec = Dvec;
  a.dQacc = dQacc;
  a.Gblk = Gblk;
  a.dK = reinterpret_cast<__nv_bfloat16*>(dK);
  a.dV = reinterpret_cast<__nv_bfloat16*>(dV);
  a.plan = plan;
  a.plan_stride = plan_stride;
  a.err = err;
  const int smem = Layout::kSmemBytes;
  e = cudaFuncSetAttribute(bwd_kb_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  timer_begin(GBS_OP_BWD, st);
  bwd_kb_kernel<<<n_ctas, kThreads, smem, st>>>(tq, tk, tv, tdo, a);
  timer_end(GBS_OP_BWD, st);
  note_launch();
  return cudaGetLastError();
}

}  // namespace gbs
