// bwd_tc.cu — K3: gated attention backward (training mode) on the tcgen05
// tensor cores, with the tile sums G that give dS fused in.
//
// The gradient flows from the loss through the softmax into the selector
// scores because the gate sits inside the softmax in log form (ai.viyan.live,
// "SAS Learns Token Importance for Sparse Attention", "The Logit Injection
// Mechanism"; NeurIPS 2026 poster page of "SAS: Simple Attention
// Sparsification via End-to-End Optimization of Context Ranking", Abstract:
// every context unit stays active in training so each one receives gradient).
// With P = exp(z - LSE), dP = dO V^T, dZ = P o (dP - D), D_i = dO_i . O_i:
//   dV = P^T dO, dK = scale dZ^T Q, dQ = scale dZ K,
//   G[r, c] = sum of dZ over the (query block r, key block c) tile.
// dS[r, c'] = G[r, c'] - g[r, c'] sum_{c<r} G[r, c] is formed afterwards from G.
//
// Tiling: one CTA per (batch, kv-head, 128-key tile = two 64-key context
// blocks); K and V stay in shared memory while the CTA walks a list of the
// 64-query blocks (of any q-head of the group) that attend its keys, two
// query blocks per step (query half 0 and 1 of the step's 128 columns; the
// two may come from different q-heads, and a missing second one is masked). In training mode the list is every query block r >= the
// tile's first key block, head by head. Per step:
//   S^T = K Q^T and dP^T = V dO^T   (M=128 keys, N=128 queries, K=d; TMEM)
//   compute warps: P^T, dZ^T (bf16) back into TMEM, dZ^T into swizzled smem,
//                  per-warp sums of dZ added into G
//   dV += P^T dO, dK += dZ^T Q      (A from TMEM, B = dO / Q MN-major)
//   dQ  = dZ K                      (A = dZ^T smem MN-major, B = K MN-major;
//                                    TMEM; each warp stages its 32 x D/2 part
//                                    in the step's now-consumed Q / dO smem
//                                    stage and the TMA warp issues tensor
//                                    reduce-adds into the fp32 accumulator)
// TMEM (512 columns): R0 = S^T / P^T, R1 = dP^T / dZ^T / dQ, dV, dK. The bf16
// P^T and dZ^T of query half h are stored over the first 32 columns of that
// half's own 64 S^T / dP^T columns.
// The compute warps work in two phases per step: phase A turns S^T into P^T
// (the dV MMA starts on it), phase B turns dP^T into dZ^T (dK and dQ start).
// The next step's S^T is issued as soon as dQ is issued, so its phase A
// overlaps the drain of dQ and the dP^T MMA.
// Warps: 0-7 compute (lane quadrant w%4, query/column half w/4), 8 TMA,
// 9 TMEM allocator + MMA issuer, 10-13 dQ drain (lane quadrant w%4): the
// drain warps move dQ out of TMEM while the compute warps start the next
// step. Every mbarrier wait is bounded.
//
// Sparse and threshold modes (the gradient through the gates renormalised
// over the kept blocks A_r; the selection itself passes no gradient) run the
// same kernel over a list built by bwd_plan_kernel: per key tile, the (q-head,
// query block) pairs that keep one of the tile's two key blocks or are one of
// them. A compute warp whose (query block, key block) pair is not kept treats
// it as masked, so its P, dZ and G are 0.
#include <cuda.h>

#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace gbs {

namespace {

using namespace sm100;

constexpr int kBK = 128;         // keys per CTA
constexpr int kBQ = 128;         // queries per step
constexpr int kQStages = 2;
constexpr int kComputeWarps = 8;
constexpr int kDrainWarps = 4;  // one per TMEM lane quadrant
constexpr int kTmaWarp = kComputeWarps, kMmaWarp = kComputeWarps + 1;
constexpr int kThreads = (kComputeWarps + 2 + kDrainWarps) * 32;
constexpr int kTmemCols = 512;
constexpr uint64_t kTimeoutNs = 4000000000ull;
constexpr int kChunk = 128 * 128;  // bytes of one 64-column chunk of a 128-row tile

template <int D>
struct BLayout {
  static constexpr int kChunks = D / 64;
  static constexpr int kTile = kChunks * kChunk;  // one 128 x D bf16 tile
  static constexpr int kKOff = 0;
  static constexpr int kVOff = kKOff + kTile;
  static constexpr int kQOff = kVOff + kTile;
  static constexpr int kdOOff = kQOff + kQStages * kTile;
  static constexpr int kZOff = kdOOff + kQStages * kTile;   // dZ^T: 128 keys x 128 queries
  static constexpr int kVecOff = kZOff + 2 * kChunk;        // LSE[128], D[128] per stage
  static constexpr int kBarOff = kVecOff + kQStages * kBQ * 8;
  static constexpr int kSmemBytes = kBarOff + 256;
};

struct BBarriers {
  uint64_t kv_full;
  uint64_t q_full[kQStages];
  uint64_t staged[kQStages];  // every drain warp has staged the step's dQ in this stage
  uint64_t s_full;   // S^T of the step landed in R0
  uint64_t dp_full;  // dP^T of the step landed in R1
  uint64_t pa_full;  // P^T written (dV can start)
  uint64_t pb_full;  // dZ^T written to TMEM and smem (dK, dQ can start)
  uint64_t dq_full;
  uint64_t dq_free;
  uint64_t done;
  uint32_t tmem_base;
  int abort_flag;
};

struct BwdArgs {
  Problem p;
  const float* S;
  const float* slse;
  const float* LSE;
  const float* Dvec;
  float* dQacc;
  float* Gblk;
  __nv_bfloat16* dK;
  __nv_bfloat16* dV;
  int n_tiles;  // 128-row tiles per head (keys and queries alike)
  const uint32_t* mbits;  // kept-block bitmap (null in training mode)
  int mwords;
  const int32_t* plan;    // per-CTA step lists (null in training mode)
  int plan_stride;
  unsigned int* err;
};

// Query-block list of CTA (key tile u, batch x kv-head bk): entry 0 is the
// count, then (q-head in group << 16 | query block r) for every r >= 2u of
// every q-head that keeps key block 2u or 2u + 1, or is one of them (its
// diagonal block). One warp per CTA (id = u * BKV + bk, the attention
// kernel's block index), ballot compaction in (q-head, r) order.
__global__ void bwd_plan_kernel(const uint32_t* __restrict__ mbits, int mwords, int Nb, int n_tiles,
                                int G, int Hq, int Hkv, int BKV, int32_t* __restrict__ plan,
                                int plan_stride) {
  const int lane = threadIdx.x & 31;
  const int id = (int)(blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5));
  if (id >= n_tiles * BKV) return;
  const int u = id / BKV, bk = id % BKV;
  const int b = bk / Hkv, kvh = bk % Hkv;
  int32_t* out = plan + (size_t)id * plan_stride;
  const int cw = (2 * u) >> 5, sh = (2 * u) & 31;  // key blocks 2u, 2u+1: bits sh, sh+1
  const uint32_t lanes_below = (1u << lane) - 1u;
  int n = 0;
  for (int hh = 0; hh < G; ++hh) {
    const size_t rowbase = (size_t)(b * Hq + kvh * G + hh) * Nb;
    for (int r0 = 2 * u; r0 < Nb; r0 += 32) {
      const int r = r0 + lane;
      bool need = false;
      if (r < Nb) need = r <= 2 * u + 1 || ((__ldg(mbits + (rowbase + r) * mwords + cw) >> sh) & 3u);
      const uint32_t m = __ballot_sync(0xffffffffu, need);
      if (need) out[1 + n + __popc(m & lanes_below)] = (hh << 16) | r;
      n += __popc(m);
    }
  }
  if (lane == 0) out[0] = n;
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

enum : int { kMasked = 0, kCausal = 1, kFull = 2 };

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
bwd_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
              const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
              const __grid_constant__ CUtensorMap tmdQ, const __grid_constant__ CUtensorMap tmQ2,
              const __grid_constant__ CUtensorMap tmdO2, BwdArgs a) {
  using L = BLayout<D>;
  extern __shared__ __align__(1024) uint8_t smem[];
  if (smem_u32(smem) & 1023u) {  // the swizzled tiles need 1024-byte alignment
    if (threadIdx.x == 0) set_error(a.err, GBS_ERR_UNSUPPORTED);
    return;
  }
  BBarriers* bars = reinterpret_cast<BBarriers*>(smem + L::kBarOff);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Problem& p = a.p;

  const int BKV = p.B * p.Hkv;
  const int u = (int)(blockIdx.x / BKV);  // key tile; small u = most work, launched first
  const int bk = (int)(blockIdx.x % BKV);
  const int b = bk / p.Hkv, kvh = bk % p.Hkv;
  const int per_head = p.Nb - 2 * u;  // training: query blocks r >= 2u of each q-head
  const int32_t* list = a.plan ? a.plan + (size_t)blockIdx.x * a.plan_stride : nullptr;
  const int n_entries = list ? dcheck(__ldg(list), 0, p.G * per_head, a.err) : p.G * per_head;
  const int n_steps = (n_entries + 1) >> 1;
  // (batch x q-head row, query block) of list entry i; r = -1 past the end.
  // Step j takes entries 2j (query half 0) and 2j + 1 (query half 1).
  auto entry_at = [&](int i, int& bh, int& r) {
    int hh = 0;
    r = -1;
    if (i < n_entries) {
      if (list) {
        const int e = __ldg(list + 1 + i);
        hh = dcheck(e >> 16, 0, p.G - 1, a.err);
        r = dcheck(e & 0xffff, 2 * u, p.Nb - 1, a.err);
      } else {
        hh = i / per_head;
        r = 2 * u + i % per_head;
      }
    }
    bh = b * p.Hq + kvh * p.G + hh;
  };

  if (threadIdx.x == 0) {
    mbar_init(&bars->kv_full, 1);
    for (int s = 0; s < kQStages; ++s) {
      mbar_init(&bars->q_full[s], 1);
      mbar_init(&bars->staged[s], kDrainWarps);
    }
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->dp_full, 1);
    mbar_init(&bars->pa_full, kComputeWarps * 32);
    mbar_init(&bars->pb_full, kComputeWarps * 32);
    mbar_init(&bars->dq_full, 1);
    mbar_init(&bars->dq_free, kDrainWarps * 32);
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
  float* vecs = reinterpret_cast<float*>(smem + L::kVecOff);

  if (warp == kTmaWarp) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      prefetch_tmap(&tmdO);
      prefetch_tmap(&tmdQ);
      prefetch_tmap(&tmQ2);
      prefetch_tmap(&tmdO2);
      mbar_arrive_expect_tx(&bars->kv_full, 2 * L::kTile);
      for (int ch = 0; ch < L::kChunks; ++ch) {
        tma_load_3d(smem + L::kKOff + ch * kChunk, &tmK, &bars->kv_full, ch * 64, u * kBK, bk);
        tma_load_3d(smem + L::kVOff + ch * kChunk, &tmV, &bars->kv_full, ch * 64, u * kBK, bk);
      }
    }
    if (lane == 0) {
      // (bh, r) of the two query halves of a step, kept until its dQ is reduced
      struct Halves {
        int bh0, r0, bh1, r1;
      };
      auto halves_of = [&](int j) {
        Halves h;
        entry_at(2 * j, h.bh0, h.r0);
        entry_at(2 * j + 1, h.bh1, h.r1);
        return h;
      };
      // adds step jj's staged dQ (8 warps x 32 rows x D/2 columns) into the accumulator
      auto reduce_step = [&](int jj, const Halves& e) -> bool {
        const int sj = jj % kQStages;
        if (!mbar_wait(&bars->staged[sj], (jj / kQStages) & 1, abort_flag, a.err, kTimeoutNs))
          return false;
        const int bh0 = e.bh0, r0 = e.r0, bh1 = e.bh1, r1 = e.r1;
#pragma unroll 1
        for (int w = 0; w < kComputeWarps; ++w) {
          // dQ rows of lane quadrant `quad` = query half quad / 2; `hq` = column half of D
          const int quad = w & 3, hq = w >> 2;
          const int r = (quad >> 1) ? r1 : r0, bh = (quad >> 1) ? bh1 : bh0;
          if (r < 0) continue;
          const int qrow0 = r * 64 + (quad & 1) * 32;
          const uint8_t* stg =
              smem + (hq == 0 ? L::kQOff : L::kdOOff) + sj * L::kTile + quad * (D / 2) * 128;
          for (int bx = 0; bx < D / 64; ++bx)
            tma_reduce_add_2d(&tmdQ, hq * (D / 2) + bx * 32, bh * p.N + qrow0, stg + bx * 4096);
        }
        bulk_commit_group();
        return true;
      };
      int issued = 0;
      bool ok = true;
      static_assert(kQStages == 2, "the producer keeps the halves of the last two steps");
      Halves prev2{0, -1, 0, -1}, prev1{0, -1, 0, -1};
      for (int j = 0; j < n_steps; ++j) {
        const int st = j % kQStages;
        const Halves cur = halves_of(j);  // list reads overlap the wait below
        // the stage is free once step j-2's MMAs are done and its staged dQ was read
        if (j >= kQStages) {
          if (!reduce_step(j - kQStages, prev2)) {
            ok = false;
            break;
          }
          bulk_wait_group_read0();
        }
        const int bh0 = cur.bh0, r0 = cur.r0, bh1 = cur.bh1, r1 = cur.r1;
        const int nv = 1 + (r1 >= 0);  // entry 2j always exists
        float* lse_s = vecs + st * 2 * kBQ;
        mbar_arrive_expect_tx(&bars->q_full[st], 2 * L::kTile + nv * 2 * 64 * 4);
        uint8_t* qs = smem + L::kQOff + st * L::kTile;
        uint8_t* ds = smem + L::kdOOff + st * L::kTile;
        if (r1 == r0 + 1 && bh1 == bh0) {
          // two consecutive blocks of one head: 128-row boxes
          for (int ch = 0; ch < L::kChunks; ++ch) {
            tma_load_3d(qs + ch * kChunk, &tmQ2, &bars->q_full[st], ch * 64, r0 * 64, bh0);
            tma_load_3d(ds + ch * kChunk, &tmdO2, &bars->q_full[st], ch * 64, r0 * 64, bh0);
          }
          const size_t off = (size_t)bh0 * p.N + r0 * 64;
          bulk_load(lse_s, a.LSE + off, kBQ * 4, &bars->q_full[st]);
          bulk_load(lse_s + kBQ, a.Dvec + off, kBQ * 4, &bars->q_full[st]);
        } else for (int h2 = 0; h2 < 2; ++h2) {
          // a missing query half (only ever half 1) repeats half 0's finite
          // rows; its warps mask it and its dQ is never reduced
          const bool own = h2 == 0 || r1 >= 0;
          const int row = (own && h2 ? r1 : r0) * 64, hd = own && h2 ? bh1 : bh0;
          for (int ch = 0; ch < L::kChunks; ++ch) {
            tma_load_3d(qs + ch * kChunk + h2 * (kChunk / 2), &tmQ, &bars->q_full[st], ch * 64, row, hd);
            tma_load_3d(ds + ch * kChunk + h2 * (kChunk / 2), &tmdO, &bars->q_full[st], ch * 64, row, hd);
          }
          if (own) {
            const size_t off = (size_t)hd * p.N + row;
            bulk_load(lse_s + h2 * 64, a.LSE + off, 64 * 4, &bars->q_full[st]);
            bulk_load(lse_s + kBQ + h2 * 64, a.Dvec + off, 64 * 4, &bars->q_full[st]);
          }
        }
        issued = j + 1;
        prev2 = prev1;
        prev1 = cur;
      }
      if (ok && n_steps >= 2) ok = reduce_step(n_steps - 2, prev2);
      if (ok) reduce_step(n_steps - 1, prev1);
      bulk_wait_group0();  // reductions reach global memory before the CTA exits
      if (*abort_flag) {
        // let loads still in flight land before the CTA exits
        mbar_drain(&bars->kv_full, 0, 1000000ull);
        for (int j = issued - kQStages < 0 ? 0 : issued - kQStages; j < issued; ++j)
          mbar_drain(&bars->q_full[j % kQStages], (j / kQStages) & 1, 1000000ull);
      }
    }
  } else if (warp == kMmaWarp) {
    // -------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idST = idesc_bf16_f32(kBK, kBQ, 0, 0);  // S^T, dP^T
      constexpr uint32_t idKV = idesc_bf16_f32(kBK, D, 1, 0);    // dV, dK (A in TMEM)
      constexpr uint32_t idQ = idesc_bf16_f32(kBQ, D, 1, 1);     // dQ (A, B MN-major)
      const uint32_t R0 = tmem, R1 = tmem + 128, TdV = tmem + 256, TdK = tmem + 384;
      const uint32_t k_addr = smem_u32(smem + L::kKOff), v_addr = smem_u32(smem + L::kVOff);
      const uint32_t z_addr = smem_u32(smem + L::kZOff);
      bool ok = mbar_wait(&bars->kv_full, 0, abort_flag, a.err, kTimeoutNs);
      // S^T_j = K Q_j^T -> R0 (waits for the step's Q / dO / LSE / D)
      auto issue_s = [&](int j) -> bool {
        const int st = j % kQStages;
        if (!mbar_wait(&bars->q_full[st], (j / kQStages) & 1, abort_flag, a.err, kTimeoutNs))
          return false;
        tc_fence_after();
        const uint32_t q_addr = smem_u32(smem + L::kQOff + st * L::kTile);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const int ch = ks >> 2, kk = ks & 3;
          mma_ss(R0, sdesc_sw128(k_addr + ch * kChunk + kk * 32, 16, 1024),
                 sdesc_sw128(q_addr + ch * kChunk + kk * 32, 16, 1024), idST, ks > 0 ? 1u : 0u);
        }
        mma_commit(&bars->s_full);
        return true;
      };
      // dP^T_j = V dO_j^T -> R1
      auto issue_dp = [&](int j) {
        const int st = j % kQStages;
        const uint32_t do_addr = smem_u32(smem + L::kdOOff + st * L::kTile);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const int ch = ks >> 2, kk = ks & 3;
          mma_ss(R1, sdesc_sw128(v_addr + ch * kChunk + kk * 32, 16, 1024),
                 sdesc_sw128(do_addr + ch * kChunk + kk * 32, 16, 1024), idST, ks > 0 ? 1u : 0u);
        }
        mma_commit(&bars->dp_full);
      };
      if (ok) ok = issue_s(0);
      if (ok) issue_dp(0);
      for (int j = 0; ok && j < n_steps; ++j) {
        const int st = j % kQStages;
        const uint32_t q_addr = smem_u32(smem + L::kQOff + st * L::kTile);
        const uint32_t do_addr = smem_u32(smem + L::kdOOff + st * L::kTile);
        // P^T / dZ^T of query half hq sit in columns [64 hq, 64 hq + 32) of R0 / R1
        if (!mbar_wait(&bars->pa_full, j & 1, abort_flag, a.err, kTimeoutNs)) break;
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < kBQ / 16; ++ks) {
          const uint32_t acol = (ks >> 2) * 64 + (ks & 3) * 8;
          mma_ts(TdV, R0 + acol, sdesc_sw128(do_addr + ks * 2048, kChunk, 1024), idKV,
                 (j > 0 || ks > 0) ? 1u : 0u);
        }
        if (!mbar_wait(&bars->pb_full, j & 1, abort_flag, a.err, kTimeoutNs)) break;
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < kBQ / 16; ++ks) {
          const uint32_t acol = (ks >> 2) * 64 + (ks & 3) * 8;
          mma_ts(TdK, R1 + acol, sdesc_sw128(q_addr + ks * 2048, kChunk, 1024), idKV,
                 (j > 0 || ks > 0) ? 1u : 0u);
        }
        // dQ_j = dZ_j K -> R1 (after dK_j has read dZ^T from R1: MMAs run in order)
#pragma unroll
        for (int ks = 0; ks < kBK / 16; ++ks)
          mma_ss(R1, sdesc_sw128(z_addr + ks * 2048, kChunk, 1024),
                 sdesc_sw128(k_addr + ks * 2048, kChunk, 1024), idQ, ks > 0 ? 1u : 0u);
        mma_commit(&bars->dq_full);
        if (j + 1 < n_steps) {
          if (!issue_s(j + 1)) break;  // R0 is free once dV_j has read P^T_j
          if (!mbar_wait(&bars->dq_free, j & 1, abort_flag, a.err, kTimeoutNs)) break;
          tc_fence_after();
          issue_dp(j + 1);  // R1 is free once dQ_j has been drained
        }
      }
      mma_commit(&bars->done);
      // after an abort the flag cuts the wait short: drain the MMAs still in
      // flight before tensor memory is freed
      if (!mbar_wait(&bars->done, 0, abort_flag, a.err, kTimeoutNs))
        mbar_drain(&bars->done, 0, 1000000ull);
    }
  } else if (warp < kComputeWarps) {
    // ------------------------------------------------------- compute warps
    const int quad = warp & 3, hq = warp >> 2;
    const int krow = quad * 32 + lane;  // key row within the tile == TMEM lane
    const int cj = 2 * u + (krow >> 6), jloc = krow & 63;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const float sc = p.scale_log2;
    uint8_t* zrow = smem + L::kZOff + hq * kChunk + krow * 128;
    bool ok = true;
    for (int j = 0; j < n_steps; ++j) {
      const int st = j % kQStages;
      int bh, r;
      entry_at(2 * j + hq, bh, r);  // this warp's query block (query half hq)
      const size_t row = (size_t)bh * p.Nb + r;
      int mode = kFull;
      float bias2 = 0.f;
      if (r < 0 || cj >= p.Nb || cj > r) {
        mode = kMasked;
      } else if (cj == r) {
        mode = kCausal;
      } else if (a.mbits && !((__ldg(a.mbits + row * a.mwords + (cj >> 5)) >> (cj & 31)) & 1u)) {
        mode = kMasked;  // key block not kept for this query block
      } else {
        bias2 = (__ldg(a.S + row * p.Nb + cj) - __ldg(a.slse + row)) * GBS_LOG2E;
      }
      if (!mbar_wait(&bars->s_full, j & 1, abort_flag, a.err, kTimeoutNs) ||
          !mbar_wait(&bars->q_full[st], (j / kQStages) & 1, abort_flag, a.err, kTimeoutNs)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const float* lse_s = vecs + st * 2 * kBQ + hq * 64;  // natural-log LSE
      const float* dvec_s = lse_s + kBQ;                   // D = dO . O
      const f32x2 scv = f2_make(sc, sc), biasv = f2_make(bias2, bias2);
      const f32x2 nlog2e = f2_make(-GBS_LOG2E, -GBS_LOG2E);
      // phase A: P^T = exp2(scale log2e s + bias - LSE log2e) from S^T alone
      float pr[64];
#pragma unroll
      for (int c = 0; c < 2; ++c) {  // two chunks of 32 query columns
        uint32_t sv[32], pp[16];
        tmem_ld32(tmem + lane_off + hq * 64 + c * 32, sv);
        tmem_wait_ld();
        if (mode == kMasked) {
#pragma unroll
          for (int k = 0; k < 32; ++k) pr[c * 32 + k] = 0.f;
        } else {
#pragma unroll
          for (int k = 0; k < 32; k += 4) {
            const float4 l4 = *reinterpret_cast<const float4*>(lse_s + c * 32 + k);
#pragma unroll
            for (int e = 0; e < 4; e += 2) {
              const int i = k + e;
              f32x2 x2 = f2_fma(f2_make(__uint_as_float(sv[i]), __uint_as_float(sv[i + 1])), scv, biasv);
              x2 = f2_fma(e == 0 ? f2_make(l4.x, l4.y) : f2_make(l4.z, l4.w), nlog2e, x2);
              float x0, x1;
              f2_split(x2, x0, x1);
              if (mode == kCausal) {
                if (c * 32 + i < jloc) x0 = -INFINITY;
                if (c * 32 + i + 1 < jloc) x1 = -INFINITY;
              }
              pr[c * 32 + i] = ex2(x0);
              pr[c * 32 + i + 1] = ex2(x1);
            }
          }
        }
#pragma unroll
        for (int k = 0; k < 16; ++k) pp[k] = pack_bf16(pr[c * 32 + 2 * k], pr[c * 32 + 2 * k + 1]);
        // bf16 P^T stays inside this warp's own 64 S^T columns, over ones already read
        tmem_st16(tmem + lane_off + hq * 64 + c * 16, pp);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bars->pa_full);
      // phase B: dZ^T = P^T o (dP^T - D)
      if (!mbar_wait(&bars->dp_full, j & 1, abort_flag, a.err, kTimeoutNs)) {
        ok = false;
        break;
      }
      tc_fence_after();
      f32x2 g2 = f2_make(0.f, 0.f);
#pragma unroll
      for (int c = 0; c < 4; ++c) {  // four chunks of 16 query columns
        uint32_t dv[16], zz[8];
        tmem_ld16(tmem + 128 + lane_off + hq * 64 + c * 16, dv);
        tmem_wait_ld();
        if (mode == kMasked) {
#pragma unroll
          for (int k = 0; k < 8; ++k) zz[k] = 0u;
        } else {
#pragma unroll
          for (int k = 0; k < 16; k += 4) {
            const float4 d4 = *reinterpret_cast<const float4*>(dvec_s + c * 16 + k);
#pragma unroll
            for (int e = 0; e < 4; e += 2) {
              const int i = k + e;
              const f32x2 dd = f2_sub(f2_make(__uint_as_float(dv[i]), __uint_as_float(dv[i + 1])),
                                      e == 0 ? f2_make(d4.x, d4.y) : f2_make(d4.z, d4.w));
              const f32x2 dz = f2_mul(f2_make(pr[c * 16 + i], pr[c * 16 + i + 1]), dd);
              g2 = f2_add(g2, dz);
              float dz0, dz1;
              f2_split(dz, dz0, dz1);
              zz[i / 2] = pack_bf16(dz0, dz1);
            }
          }
        }
        // dZ^T of keys' query columns [16 c, 16 c + 16) -> packed columns [8 c, 8 c + 8)
        // of this warp's 64 dP^T columns, all already read by chunks 0..c
        tmem_st8(tmem + 128 + lane_off + hq * 64 + c * 8, zz);
#pragma unroll
        for (int gi = 0; gi < 2; ++gi) {
          const int gg = c * 2 + gi;
          *reinterpret_cast<uint4*>(zrow + ((gg ^ (krow & 7)) << 4)) =
              make_uint4(zz[4 * gi], zz[4 * gi + 1], zz[4 * gi + 2], zz[4 * gi + 3]);
        }
      }
      tmem_wait_st();
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&bars->pb_full);
      float g, g_hi;
      f2_split(g2, g, g_hi);
      g = warp_sum(g + g_hi);
      if (lane == 0 && mode != kMasked) atomicAdd(a.Gblk + ((size_t)bh * p.Nb + r) * p.Nb + cj, g);
    }

    // epilogue: dV and dK rows of this tile (TMEM lane == key row)
    if (ok && mbar_wait(&bars->done, 0, abort_flag, a.err, kTimeoutNs)) {
      tc_fence_after();
      const int key = u * kBK + krow;
      const size_t orow = ((size_t)bk * p.N + key) * D + hq * (D / 2);
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        uint32_t ov[32], ok2[32];
        tmem_ld32(tmem + 256 + lane_off + hq * (D / 2) + c * 32, ov);
        tmem_ld32(tmem + 384 + lane_off + hq * (D / 2) + c * 32, ok2);
        tmem_wait_ld();
        if (key < p.N) {
          uint4* dvp = reinterpret_cast<uint4*>(a.dV + orow + c * 32);
          uint4* dkp = reinterpret_cast<uint4*>(a.dK + orow + c * 32);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            dvp[k] = make_uint4(
                pack_bf16(__uint_as_float(ov[8 * k]), __uint_as_float(ov[8 * k + 1])),
                pack_bf16(__uint_as_float(ov[8 * k + 2]), __uint_as_float(ov[8 * k + 3])),
                pack_bf16(__uint_as_float(ov[8 * k + 4]), __uint_as_float(ov[8 * k + 5])),
                pack_bf16(__uint_as_float(ov[8 * k + 6]), __uint_as_float(ov[8 * k + 7])));
            const float s = p.scale;
            dkp[k] = make_uint4(
                pack_bf16(__uint_as_float(ok2[8 * k]) * s, __uint_as_float(ok2[8 * k + 1]) * s),
                pack_bf16(__uint_as_float(ok2[8 * k + 2]) * s, __uint_as_float(ok2[8 * k + 3]) * s),
                pack_bf16(__uint_as_float(ok2[8 * k + 4]) * s, __uint_as_float(ok2[8 * k + 5]) * s),
                pack_bf16(__uint_as_float(ok2[8 * k + 6]) * s, __uint_as_float(ok2[8 * k + 7]) * s));
          }
        }
      }
    }
  } else {
    // ------------------------------------------------------- dQ drain warps
    const int quad = warp & 3;  // TMEM lane quadrant == 32 query rows of dQ
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    for (int j = 0; j < n_steps; ++j) {
      const int st = j % kQStages;
      if (!mbar_wait(&bars->dq_full, j & 1, abort_flag, a.err, kTimeoutNs)) break;
      tc_fence_after();
      // 32 rows x D columns as 32 x 32 fp32 boxes (128-byte swizzle): columns
      // [0, D/2) go to the step's Q stage, [D/2, D) to its dO stage; every MMA
      // of the step has finished reading both
#pragma unroll
      for (int bx = 0; bx < D / 32; ++bx) {
        const int hq = bx / (D / 64), sub = bx % (D / 64);
        uint8_t* row = smem + (hq == 0 ? L::kQOff : L::kdOOff) + st * L::kTile +
                       quad * (D / 2) * 128 + sub * 4096 + lane * 128;
        uint32_t o[32];
        tmem_ld32(tmem + 128 + lane_off + bx * 32, o);
        tmem_wait_ld();
#pragma unroll
        for (int gi = 0; gi < 8; ++gi)
          *reinterpret_cast<uint4*>(row + ((gi ^ (lane & 7)) << 4)) =
              make_uint4(o[4 * gi], o[4 * gi + 1], o[4 * gi + 2], o[4 * gi + 3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&bars->dq_free);  // R1 is free; the reduction proceeds from smem
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->staged[st]);  // the TMA warp issues the reduction
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// dQ = scale * dQacc, rounded to bf16 (8 elements per thread).
__global__ void dq_convert_kernel(const float* __restrict__ acc, __nv_bfloat16* __restrict__ dQ,
                                  float scale, size_t n8) {
  const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n8) return;
  const float4 a = reinterpret_cast<const float4*>(acc)[2 * i];
  const float4 c = reinterpret_cast<const float4*>(acc)[2 * i + 1];
  reinterpret_cast<uint4*>(dQ)[i] =
      make_uint4(pack_bf16(a.x * scale, a.y * scale), pack_bf16(a.z * scale, a.w * scale),
                 pack_bf16(c.x * scale, c.y * scale), pack_bf16(c.z * scale, c.w * scale));
}

// D_i = dO_i . O_i, one warp per row, 16-byte loads.
template <int D>
__global__ void dot_rows_kernel(const __nv_bfloat16* __restrict__ O,
                                const __nv_bfloat16* __restrict__ dO, float* __restrict__ Dvec,
                                size_t rows) {
  const size_t row = (size_t)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  float s = 0.f;
  if (lane < D / 8) {
    const uint4 x = reinterpret_cast<const uint4*>(O + row * D)[lane];
    const uint4 y = reinterpret_cast<const uint4*>(dO + row * D)[lane];
    const __nv_bfloat162* xh = reinterpret_cast<const __nv_bfloat162*>(&x);
    const __nv_bfloat162* yh = reinterpret_cast<const __nv_bfloat162*>(&y);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 xf = __bfloat1622float2(xh[k]), yf = __bfloat1622float2(yh[k]);
      s = fmaf(xf.x, yf.x, fmaf(xf.y, yf.y, s));
    }
  }
  s = warp_sum(s);
  if (lane == 0) Dvec[row] = s;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

bool make_map128(CUtensorMap* m, const void* base, int d, int rows, int heads, int box_rows = 128) {
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

// dQ accumulator, fp32 rows of D: dims (D, rows), 32 x 32 boxes, 128-byte swizzle.
bool make_map_dq(CUtensorMap* m, const void* base, int d, size_t rows) {
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
  const cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)d * 4};
  const cuuint32_t box[2] = {32, 32};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D>
cudaError_t launch_bwd_typed(const BwdArgs& a, const void* Q, const void* K, const void* V,
                             const void* O, const void* dO, void* dQ, cudaStream_t st) {
  const Problem& p = a.p;
  const size_t rows = (size_t)p.B * p.Hq * p.N;
  dot_rows_kernel<D><<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(
      (const __nv_bfloat16*)O, (const __nv_bfloat16*)dO, const_cast<float*>(a.Dvec), rows);
  note_launch();
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  CUtensorMap tq, tk, tv, tdo, tdq, tq2, tdo2;
  if (!make_map128(&tq, Q, D, p.N, p.B * p.Hq, 64) || !make_map128(&tk, K, D, p.N, p.B * p.Hkv) ||
      !make_map128(&tv, V, D, p.N, p.B * p.Hkv) || !make_map128(&tdo, dO, D, p.N, p.B * p.Hq, 64) ||
      !make_map128(&tq2, Q, D, p.N, p.B * p.Hq) || !make_map128(&tdo2, dO, D, p.N, p.B * p.Hq) ||
      !make_map_dq(&tdq, a.dQacc, D, rows))
    return cudaErrorInvalidValue;
  auto kern = bwd_tc_kernel<D>;
  const int smem = BLayout<D>::kSmemBytes;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const unsigned grid = (unsigned)(p.B * p.Hkv * a.n_tiles);
  timer_begin(GBS_OP_BWD, st);
  kern<<<grid, kThreads, smem, st>>>(tq, tk, tv, tdo, tdq, tq2, tdo2, a);
  timer_end(GBS_OP_BWD, st);
  note_launch();
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const size_t n8 = rows * D / 8;
  dq_convert_kernel<<<(unsigned)((n8 + 255) / 256), 256, 0, st>>>(a.dQacc, (__nv_bfloat16*)dQ,
                                                                    p.scale, n8);
  note_launch();
  return cudaGetLastError();
}

}  // namespace

bool bwd_tc_supported(const Problem& p) {
  return p.dtype == GBS_BF16 && p.bs == 64 && (p.d == 64 || p.d == 128) && p.N % 64 == 0 &&
         p.Nb <= 65536;
}

size_t bwd_plan_ints(const Problem& p) {
  if (p.mode == GBS_TRAIN) return 0;
  const size_t n_tiles = (size_t)(p.Nb + 1) / 2;
  return (size_t)p.B * p.Hkv * n_tiles * (1 + (size_t)p.G * p.Nb);
}

cudaError_t launch_bwd_tc(const Problem& p, const void* Q, const void* K, const void* V,
                          const float* S, const float* slse, const void* O, const float* LSE,
                          const void* dO, void* dQ, void* dK, void* dV, float* Dvec, float* Gblk,
                          float* dQacc, const uint32_t* mbits, int mwords, int32_t* plan,
                          unsigned int* err, cudaStream_t st) {
  if (!bwd_tc_supported(p)) return cudaErrorNotSupported;
  const bool sparse = p.mode != GBS_TRAIN;
  if (sparse && (!mbits || !plan)) return cudaErrorInvalidValue;
  BwdArgs a;
  a.p = p;
  a.S = S;
  a.slse = slse;
  a.LSE = LSE;
  a.Dvec = Dvec;
  a.dQacc = dQacc;
  a.Gblk = Gblk;
  a.dK = reinterpret_cast<__nv_bfloat16*>(dK);
  a.dV = reinterpret_cast<__nv_bfloat16*>(dV);
  a.n_tiles = (p.Nb + 1) / 2;
  a.mbits = sparse ? mbits : nullptr;
  a.mwords = mwords;
  a.plan = sparse ? plan : nullptr;
  a.plan_stride = 1 + p.G * p.Nb;
  a.err = err;
  if (sparse) {
    const int ctas = p.B * p.Hkv * a.n_tiles;
    bwd_plan_kernel<<<(unsigned)((ctas + 7) / 8), 256, 0, st>>>(
        mbits, mwords, p.Nb, a.n_tiles, p.G, p.Hq, p.Hkv, p.B * p.Hkv, plan, a.plan_stride);
    note_launch();
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  cudaError_t e = cudaMemsetAsync(dQacc, 0, (size_t)p.B * p.Hq * p.N * p.d * sizeof(float), st);
  if (e == cudaSuccess)
    e = cudaMemsetAsync(Gblk, 0, (size_t)p.B * p.Hq * p.Nb * p.Nb * sizeof(float), st);
  if (e != cudaSuccess) return e;
  if (p.d == 64) return launch_bwd_typed<64>(a, Q, K, V, O, dO, dQ, st);
  return launch_bwd_typed<128>(a, Q, K, V, O, dO, dQ, st);
}

}  // namespace gbs
