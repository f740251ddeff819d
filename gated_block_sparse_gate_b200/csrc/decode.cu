// decode.cu — K4: sparse one-token decode, split over the selected blocks.
//
// One query per sequence sits at position L-1; its current block
// cur = (L-1)/64 is always attended (bias 0, keys up to L-1) and the historical
// blocks are the Top-K list of K1 with gates renormalised over it (NeurIPS
// 2026 poster page of "SAS: Simple Attention Sparsification via End-to-End
// Optimization of Context Ranking", Abstract: a fixed budget of context units
// per query; Hugging Face paper page, Abstract: the current block is always
// retained).
//
// The work is bound by HBM: every selected block streams 64 keys and 64 values
// once. Split kernel: grid (B*Hq, splits); each CTA takes a contiguous share of
// the (selected + current) block list; a group of D/8 lanes owns one key row
// and loads it with 16-byte vector loads (for bf16 the block's eight key and
// eight value rows of a lane are all in flight before any arithmetic; fp32
// loads the values after the scores), reduces the dot product with shuffles
// and keeps an online
// softmax state. The CTA merges its eight groups and writes one partial
// (m, l, acc[D]) per split; the combine kernel merges the splits.
//
// Serving layouts (gbs_decode_ex): the cache may sit on 64-token pages found
// through a block table, each sequence may have its own length, and with
// group-shared selection one CTA serves two q-heads of a kv group, so each
// row it loads feeds both. That variant is bound by instruction issue, not
// bytes, so with d = 128 a lane's 16 dot-product partials (8 rows x 2 heads)
// are reduced across its 16-lane group by one butterfly (15 shuffles), each
// lane then takes one exponential, and the products run on packed fp32 pairs.
// A CTA resolves the addresses of up to 64 of its blocks at once (index, gate,
// page) before it streams them.
#include "common.cuh"
#include "internal.h"

namespace gbs {

namespace {

constexpr int kBS = 64;
constexpr int kThreads = 128;
constexpr int kEntChunk = 64;  // selected blocks whose addresses are resolved at once

struct Vec8 {
  float v[8];
};

template <typename T>
__device__ __forceinline__ Vec8 load8(const T* ptr);

template <>
__device__ __forceinline__ Vec8 load8<__nv_bfloat16>(const __nv_bfloat16* ptr) {
  const uint4 u = __ldg(reinterpret_cast<const uint4*>(ptr));
  Vec8 r;
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(h[i]);
    r.v[2 * i] = f.x;
    r.v[2 * i + 1] = f.y;
  }
  return r;
}

template <>
__device__ __forceinline__ Vec8 load8<float>(const float* ptr) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(ptr));
  const float4 b = __ldg(reinterpret_cast<const float4*>(ptr) + 1);
  Vec8 r;
  r.v[0] = a.x; r.v[1] = a.y; r.v[2] = a.z; r.v[3] = a.w;
  r.v[4] = b.x; r.v[5] = b.y; r.v[6] = b.z; r.v[7] = b.w;
  return r;
}

// Element i of eight bf16 values held as one 16-byte word (element 0 in the
// low half of .x); a bf16 widens to fp32 by a 16-bit shift.
__device__ __forceinline__ float bf16_elem(const uint4& u, int i) {
  const uint32_t w = i < 2 ? u.x : (i < 4 ? u.y : (i < 6 ? u.z : u.w));
  return __uint_as_float((i & 1) ? (w & 0xffff0000u) : (w << 16));
}

// packed fp32 pairs (one 64-bit register, two lanes of arithmetic per instruction)
struct F2 { uint64_t v; };
__device__ __forceinline__ F2 mk2(float lo, float hi) {
  F2 r; asm("mov.b64 %0, {%1, %2};" : "=l"(r.v) : "f"(lo), "f"(hi)); return r;
}
__device__ __forceinline__ F2 f2m(float a0, float a1, float b0, float b1) {
  F2 r; asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r.v) : "l"(mk2(a0, a1).v), "l"(mk2(b0, b1).v)); return r;
}
__device__ __forceinline__ F2 f2fma(float a0, float a1, float b0, float b1, F2 c) {
  F2 r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r.v) : "l"(mk2(a0, a1).v), "l"(mk2(b0, b1).v), "l"(c.v));
  return r;
}
__device__ __forceinline__ float f2sum(F2 x) {
  float lo, hi; asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(x.v)); return lo + hi;
}
__device__ __forceinline__ void f2acc8(float (&acc)[8], float p, const float (&v)[8]) {
#pragma unroll
  for (int i = 0; i < 8; i += 2) {
    F2 r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r.v) : "l"(mk2(p, p).v), "l"(mk2(v[i], v[i + 1]).v),
        "l"(mk2(acc[i], acc[i + 1]).v));
    asm("mov.b64 {%0, %1}, %2;" : "=f"(acc[i]), "=f"(acc[i + 1]) : "l"(r.v));
  }
}

// Online-softmax state of one lane group (log2 domain).
struct State {
  float m, l, acc[8];
};

// While a block is computed the next block's key and value rows are
// prefetched into L2 (one line per thread and tensor), so its row loads wait
// on L2 rather than on HBM: split kernel 0.141 -> 0.131 ms (group-shared) and
// 0.324 -> 0.316 ms (per-head) on 64 sequences x 131072, results unchanged.
// In the group-shared bf16 path the key rows of the next block are requested
// into the key registers as soon as the current block's dot products have
// consumed them (0.131 -> 0.125 ms).
//
// Grid: x = CTA row (one selection row, or a slice of NH q-heads of a
// group-shared selection row), y = split. Each CTA handles NH q-heads that
// share one selection and one kv head, so every key and value row it loads
// serves all NH of them. With NH = 2 the registers are capped for four CTAs
// per SM (no spills), which keeps enough rows in flight.
template <typename T, int D, int NH>
__global__ void __launch_bounds__(kThreads, NH == 2 ? 4 : 1)
decode_split_kernel(Problem p, const T* __restrict__ q, const T* __restrict__ Kc,
                    const T* __restrict__ Vc, Selection sel, KvLayout kv, int grouped, int n_sub,
                    int splits, float* __restrict__ part_ml, float* __restrict__ part_acc) {
  constexpr int LPK = D / 8;             // lanes per key row
  constexpr int GPW = 32 / LPK;          // key groups per warp
  constexpr int NGROUPS = (kThreads / 32) * GPW;
  constexpr int ROWS_PER_GROUP = kBS / NGROUPS;
  constexpr bool kRaw = sizeof(T) == 2;
  __shared__ float s_m[NGROUPS][NH], s_l[NGROUPS][NH];
  __shared__ float s_acc[NGROUPS][NH][D];
  __shared__ int s_row0[kEntChunk];  // first cache row (units of D elements); -1: skip it
  __shared__ float s_bias[kEntChunk];
  __shared__ int s_rows[kEntChunk];

  const int srow = blockIdx.x / n_sub, slice = blockIdx.x % n_sub, split = blockIdx.y;
  int b, kvh, h0;
  if (grouped) {
    b = srow / p.Hkv;
    kvh = srow % p.Hkv;
    h0 = kvh * p.G + slice * NH;
  } else {
    b = srow / p.Hq;
    h0 = srow % p.Hq;
    kvh = h0 / p.G;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int grp_in_warp = lane / LPK, sub = lane % LPK;
  const int group = warp * GPW + grp_in_warp;
  int L = p.N;
  if (kv.seq_lens) {  // a length outside [1, N] is clamped here and reported by the combine
    L = __ldg(kv.seq_lens + b);
    L = L < 1 ? 1 : (L > p.N ? p.N : L);
  }
  const int cur = (L - 1) / kBS;
  const int n_hist = dcheck(sel.cnt[srow], 0, min(p.topk, cur), kv.err);
  const int n_ent = n_hist + 1;  // + current block
  const int per = (n_ent + splits - 1) / splits;
  const int e0 = split * per, e1 = min(n_ent, e0 + per);

  Vec8 qv[NH];
#pragma unroll
  for (int g = 0; g < NH; ++g) {
    qv[g] = load8<T>(q + ((size_t)b * p.Hq + h0 + g) * D + sub * 8);
#pragma unroll
    for (int i = 0; i < 8; ++i) qv[g].v[i] *= p.scale_log2;
  }
  State st[NH];
#pragma unroll
  for (int g = 0; g < NH; ++g) {
    st[g].m = -INFINITY;
    st[g].l = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) st[g].acc[i] = 0.f;
  }

  const int contig = (b * p.Hkv + kvh) * p.N;  // first row of this kv head's cache
  constexpr bool kPipeK = kRaw && NH == 2 && LPK == 16;
  uint4 kr_next[kPipeK ? ROWS_PER_GROUP : 1];
  bool have_k = false;  // kr_next holds the key rows of the block about to be processed
  for (int cs = e0; cs < e1; cs += kEntChunk) {
    const int ce = min(e1, cs + kEntChunk);
    // resolve the chunk's blocks (index, gate, page) in parallel, so the block
    // loop below starts each block's row loads without a dependent lookup
    __syncthreads();
    for (int t = threadIdx.x; t < ce - cs; t += kThreads) {
      const int e = cs + t;
      const bool is_cur = e == n_hist;
      const int c = is_cur ? cur : dcheck(sel.idx[(size_t)srow * p.topk + e], 0, cur - 1, kv.err);
      int row0 = contig + c * kBS;
      if (kv.btab) {
        const int page = __ldg(kv.btab + (size_t)b * kv.max_blocks + c);
        if (page < 0 || page >= kv.num_pages) {
          set_error(kv.err, GBS_ERR_INVALID_ARG);
          row0 = -1;
        } else {
          row0 = (page * p.Hkv + kvh) * kBS;
        }
      }
      s_row0[t] = row0;
      s_bias[t] = is_cur ? 0.f : sel.logg[(size_t)srow * p.topk + e] * GBS_LOG2E;
      s_rows[t] = is_cur ? L - cur * kBS : kBS;  // rows of the block inside the sequence
    }
    __syncthreads();
  for (int e = cs; e < ce; ++e) {
    if (s_row0[e - cs] < 0) continue;  // a page outside the pool: skipped, reported
    const size_t base = (size_t)s_row0[e - cs] * D;
    const float bias2 = s_bias[e - cs];
    const int nrows = s_rows[e - cs];
    if constexpr (kRaw) {
      // bring the next block's key and value rows into L2 while this one is
      // computed: one 128-byte line per thread and tensor
      if (e + 1 < ce && s_row0[e + 1 - cs] >= 0) {
        constexpr int kLinesPerRow = D * 2 / 128;
        const int n_lines = s_rows[e + 1 - cs] * kLinesPerRow;  // rows inside the sequence only
        const size_t nb = (size_t)s_row0[e + 1 - cs] * D;
        for (int t = threadIdx.x; t < n_lines; t += kThreads) {
          asm volatile("prefetch.global.L2 [%0];" ::"l"(Kc + nb + (size_t)t * 64));
          asm volatile("prefetch.global.L2 [%0];" ::"l"(Vc + nb + (size_t)t * 64));
        }
      }
    }
    // rows handled by this group inside the block
    const int row0 = group * ROWS_PER_GROUP;
    float s[NH][ROWS_PER_GROUP];
    if constexpr (kRaw && NH == 2 && LPK == 16) {
      // bf16, two q-heads, 16 lanes a row: the 16 dot-product partials of a
      // lane (8 rows x 2 heads) are reduced across the group by a butterfly that
      // halves the values a lane keeps at offsets 8, 4, 2, 1, so lane `sub`
      // ends with the full dot product of head sub / 8, row sub % 8 (15 shuffles
      // instead of 16 four-level reductions). Each lane then takes one
      // exponential; row maxima and sums reduce over the head's 8 lanes, and the
      // PV update broadcasts each row's probability from its lane.
      uint4 vr[ROWS_PER_GROUP];
      if (!have_k) {
#pragma unroll
        for (int rr = 0; rr < ROWS_PER_GROUP; ++rr) {
          const int row = min(row0 + rr, nrows - 1);
          kr_next[rr] = __ldg(reinterpret_cast<const uint4*>(Kc + base + (size_t)row * D + sub * 8));
        }
      }
#pragma unroll
      for (int rr = 0; rr < ROWS_PER_GROUP; ++rr) {
        const int row = min(row0 + rr, nrows - 1);
        vr[rr] = __ldg(reinterpret_cast<const uint4*>(Vc + base + (size_t)row * D + sub * 8));
      }
      const uint4* kr = kr_next;
      float v[16];
#pragma unroll
      for (int rr = 0; rr < 8; ++rr) {
        float kf[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) kf[i] = bf16_elem(kr[rr], i);
#pragma unroll
        for (int g = 0; g < 2; ++g) {
          F2 acc = f2m(qv[g].v[0], qv[g].v[1], kf[0], kf[1]);
          acc = f2fma(qv[g].v[2], qv[g].v[3], kf[2], kf[3], acc);
          acc = f2fma(qv[g].v[4], qv[g].v[5], kf[4], kf[5], acc);
          acc = f2fma(qv[g].v[6], qv[g].v[7], kf[6], kf[7], acc);
          v[g * 8 + rr] = f2sum(acc);
        }
      }
#pragma unroll
      for (int st_ = 0; st_ < 4; ++st_) {
        const int off = 8 >> st_;
        const bool upper = (sub & off) != 0;
#pragma unroll
        for (int i = 0; i < off; ++i) {
          const float send = upper ? v[i] : v[i + off];
          const float keep = upper ? v[i + off] : v[i];
          v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
        }
      }
      // the key rows of this block are consumed: request the next block's into
      // the same registers, so they arrive while this block's softmax and PV run
      have_k = e + 1 < ce && s_row0[e + 1 - cs] >= 0;
      if (have_k) {
        const size_t nbase = (size_t)s_row0[e + 1 - cs] * D;
        const int nrows_n = s_rows[e + 1 - cs];
#pragma unroll
        for (int rr = 0; rr < ROWS_PER_GROUP; ++rr) {
          const int row = min(row0 + rr, nrows_n - 1);
          kr_next[rr] = __ldg(reinterpret_cast<const uint4*>(Kc + nbase + (size_t)row * D + sub * 8));
        }
      }
      const int gl = sub >> 3, rl = sub & 7;
      const float s_me = (row0 + rl < nrows) ? v[0] + bias2 : -INFINITY;
      float mx = s_me;
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
      const float m_old = gl ? st[1].m : st[0].m;
      const float m_new = mx > -INFINITY ? fmaxf(m_old, mx) : m_old;
      const float pr = mx > -INFINITY ? exp2f(s_me - m_new) : 0.f;
      float ps = pr;
      ps += __shfl_xor_sync(0xffffffffu, ps, 1);
      ps += __shfl_xor_sync(0xffffffffu, ps, 2);
      ps += __shfl_xor_sync(0xffffffffu, ps, 4);
      const float m_oth = __shfl_xor_sync(0xffffffffu, m_new, 8);
      const float ps_oth = __shfl_xor_sync(0xffffffffu, ps, 8);
#pragma unroll
      for (int g = 0; g < 2; ++g) {
        const float mn = (g == gl) ? m_new : m_oth;
        const float pg = (g == gl) ? ps : ps_oth;
        const float corr = st[g].m == mn ? 1.f : exp2f(st[g].m - mn);
        st[g].l = st[g].l * corr + pg;
#pragma unroll
        for (int i = 0; i < 8; ++i) st[g].acc[i] *= corr;
        st[g].m = mn;
      }
#pragma unroll
      for (int rr = 0; rr < 8; ++rr) {
        float vf[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) vf[i] = bf16_elem(vr[rr], i);
#pragma unroll
        for (int g = 0; g < 2; ++g) {
          const float pg = __shfl_sync(0xffffffffu, pr, g * 8 + rr, 16);
          f2acc8(st[g].acc, pg, vf);
        }
      }
    } else if constexpr (kRaw) {
      // bf16: the block's key and value rows are all requested before any
      // arithmetic (one memory latency per block), and held as raw 16-byte
      // words, which costs the registers that eight converted rows would
      uint4 kr[ROWS_PER_GROUP], vr[ROWS_PER_GROUP];
#pragma unroll
      for (int rr = 0; rr < ROWS_PER_GROUP; ++rr) {
        const int row = min(row0 + rr, nrows - 1);
        kr[rr] = __ldg(reinterpret_cast<const uint4*>(Kc + base + (size_t)row * D + sub * 8));
      }
#pragma unroll
      for (int rr = 0; rr < ROWS_PER_GROUP; ++rr) {
        const int row = min(row0 + rr, nrows - 1);
        vr[rr] = __ldg(reinterpret_cast<const uint4*>(Vc + base + (size_t)row * D + sub * 8));
      }
#pragma unroll
      for (int rr = 0; rr < ROWS_PER_GROUP; ++rr) {
#pragma unroll
        for (int g = 0; g < NH; ++g) {
          float d = 0.f;
#pragma unroll
          for (int i = 0; i < 8; ++i) d = fmaf(qv[g].v[i], bf16_elem(kr[rr], i), d);
#pragma unroll
          for (int o = LPK / 2; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
          s[g][rr] = (row0 + rr < nrows) ? d + bias2 : -INFINITY;
        }
      }
#pragma unroll
      for (int g = 0; g < NH; ++g) {
        float mloc = st[g].m;
#pragma unroll
        for (int rr = 0; rr < ROWS_PER_GROUP; ++rr) mloc = fmaxf(mloc, s[g][rr]);
        if (mloc > -INFINITY) {
          const float corr = exp2f(st[g].m - mloc);
          st[g].l *= corr;
#pragma unroll
          for (int i = 0; i < 8; ++i) st[g].acc[i] *= corr;
          st[g].m = mloc;
#pragma unroll
          for (int rr = 0; rr < ROWS_PER_GROUP; ++rr) {
            const float pr = exp2f(s[g][rr] - mloc);
            st[g].l += pr;
#pragma unroll
            for (int i = 0; i < 8; ++i) st[g].acc[i] = fmaf(pr, bf16_elem(vr[rr], i), st[g].acc[i]);
          }
        }
      }
    } else {
    Vec8 kvr[ROWS_PER_GROUP];
#pragma unroll
    for (int rr = 0; rr < ROWS_PER_GROUP; ++rr) {
      const int row = min(row0 + rr, nrows - 1);
      kvr[rr] = load8<T>(Kc + base + (size_t)row * D + sub * 8);
    }
#pragma unroll
    for (int rr = 0; rr < ROWS_PER_GROUP; ++rr) {
#pragma unroll
      for (int g = 0; g < NH; ++g) {
        float d = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) d = fmaf(qv[g].v[i], kvr[rr].v[i], d);
#pragma unroll
        for (int o = LPK / 2; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
        s[g][rr] = (row0 + rr < nrows) ? d + bias2 : -INFINITY;
      }
    }
#pragma unroll
    for (int rr = 0; rr < ROWS_PER_GROUP; ++rr) {
      const int row = min(row0 + rr, nrows - 1);
      kvr[rr] = load8<T>(Vc + base + (size_t)row * D + sub * 8);
    }
#pragma unroll
    for (int g = 0; g < NH; ++g) {
      float mloc = st[g].m;
#pragma unroll
      for (int rr = 0; rr < ROWS_PER_GROUP; ++rr) mloc = fmaxf(mloc, s[g][rr]);
      if (mloc > -INFINITY) {
        const float corr = exp2f(st[g].m - mloc);
        st[g].l *= corr;
#pragma unroll
        for (int i = 0; i < 8; ++i) st[g].acc[i] *= corr;
        st[g].m = mloc;
#pragma unroll
        for (int rr = 0; rr < ROWS_PER_GROUP; ++rr) {
          const float pr = exp2f(s[g][rr] - mloc);
          st[g].l += pr;
#pragma unroll
          for (int i = 0; i < 8; ++i) st[g].acc[i] = fmaf(pr, kvr[rr].v[i], st[g].acc[i]);
        }
      }
    }
    }
  }
  }
  // merge the groups of the CTA
#pragma unroll
  for (int g = 0; g < NH; ++g) {
    if (sub == 0) {
      s_m[group][g] = st[g].m;
      s_l[group][g] = st[g].l;
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) s_acc[group][g][sub * 8 + i] = st[g].acc[i];
  }
  __syncthreads();
  for (int k = threadIdx.x; k < NH * D; k += kThreads) {
    const int g = k / D, col = k % D;
    float M = -INFINITY;
#pragma unroll
    for (int gr = 0; gr < NGROUPS; ++gr) M = fmaxf(M, s_m[gr][g]);
    float a = 0.f;
    if (M > -INFINITY)
      for (int gr = 0; gr < NGROUPS; ++gr) a += s_acc[gr][g][col] * exp2f(s_m[gr][g] - M);
    const size_t pidx = ((size_t)b * p.Hq + h0 + g) * splits + split;
    part_acc[pidx * D + col] = a;
    if (col == 0) {
      float l = 0.f;
      if (M > -INFINITY)
        for (int gr = 0; gr < NGROUPS; ++gr) l += s_l[gr][g] * exp2f(s_m[gr][g] - M);
      part_ml[pidx * 2] = M;
      part_ml[pidx * 2 + 1] = l;
    }
  }
}

template <typename T, int D>
__global__ void decode_combine_kernel(Problem p, int splits, const float* __restrict__ part_ml,
                                      const float* __restrict__ part_acc, T* __restrict__ O,
                                      float* __restrict__ LSE, KvLayout kv) {
  const int bh = blockIdx.x;
  if (kv.seq_lens && threadIdx.x == 0) {
    const int L = __ldg(kv.seq_lens + bh / p.Hq);
    if (L < 1 || L > p.N) set_error(kv.err, GBS_ERR_INVALID_ARG);
  }
  float M = -INFINITY;
  for (int s = 0; s < splits; ++s) M = fmaxf(M, part_ml[((size_t)bh * splits + s) * 2]);
  float l = 0.f;
  for (int s = 0; s < splits; ++s) {
    const float ms = part_ml[((size_t)bh * splits + s) * 2];
    if (ms > -INFINITY) l += part_ml[((size_t)bh * splits + s) * 2 + 1] * exp2f(ms - M);
  }
  const float inv = 1.f / l;
  for (int k = threadIdx.x; k < D; k += blockDim.x) {
    float a = 0.f;
    for (int s = 0; s < splits; ++s) {
      const float ms = part_ml[((size_t)bh * splits + s) * 2];
      if (ms > -INFINITY) a += part_acc[((size_t)bh * splits + s) * D + k] * exp2f(ms - M);
    }
    O[(size_t)bh * D + k] = from_f32<T>(a * inv);
  }
  if (threadIdx.x == 0) LSE[bh] = (M + log2f(l)) * GBS_LN2;
}

template <typename T, int D, int NH>
cudaError_t decode_typed(const Problem& p, const void* q, const void* Kc, const void* Vc,
                         const Selection& sel, const KvLayout& kv, bool grouped, int splits,
                         float* part_ml, float* part_acc, void* O, float* LSE, cudaStream_t st) {
  const int n_sub = grouped ? p.G / NH : 1;
  const int rows = grouped ? p.B * p.Hkv * n_sub : p.B * p.Hq;
  timer_begin(GBS_OP_DECODE, st);
  decode_split_kernel<T, D, NH><<<dim3(rows, splits), kThreads, 0, st>>>(
      p, (const T*)q, (const T*)Kc, (const T*)Vc, sel, kv, grouped ? 1 : 0, n_sub, splits,
      part_ml, part_acc);
  timer_end(GBS_OP_DECODE, st);
  note_launch();
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  decode_combine_kernel<T, D><<<p.B * p.Hq, D, 0, st>>>(p, splits, part_ml, part_acc, (T*)O, LSE,
                                                          kv);
  note_launch();
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t decode_heads(const Problem& p, const void* q, const void* Kc, const void* Vc,
                         const Selection& sel, const KvLayout& kv, bool grouped, int splits,
                         float* part_ml, float* part_acc, void* O, float* LSE, cudaStream_t st) {
  const int nh = decode_heads_per_cta(p, grouped);
  if (nh == 2)
    return decode_typed<T, D, 2>(p, q, Kc, Vc, sel, kv, grouped, splits, part_ml, part_acc, O, LSE, st);
  return decode_typed<T, D, 1>(p, q, Kc, Vc, sel, kv, grouped, splits, part_ml, part_acc, O, LSE, st);
}

}  // namespace

int decode_resident_ctas(const Problem& p, bool grouped) {
  const int nh = decode_heads_per_cta(p, grouped);
  const void* fn = nullptr;
#define GBS_FN(T, DD)                                                                  \
  fn = nh == 2 ? (const void*)decode_split_kernel<T, DD, 2> : (const void*)decode_split_kernel<T, DD, 1>
  if (p.dtype == GBS_F32) {
    if (p.d == 64) GBS_FN(float, 64); else GBS_FN(float, 128);
  } else {
    if (p.d == 64) GBS_FN(__nv_bfloat16, 64); else GBS_FN(__nv_bfloat16, 128);
  }
#undef GBS_FN
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, fn, kThreads, 0) != cudaSuccess || n < 1)
    n = 1;
  return n;
}

int decode_heads_per_cta(const Problem& p, bool grouped) {
  // Two q-heads per CTA measured fastest on the 64 x 131072 decode with G = 4
  // (0.240 ms against 0.266 ms for one or four): one is the per-head kernel with
  // the group's CTAs sharing blocks through L2, four halves the CTAs resident
  // per SM (about 200 registers a thread) and with them the loads in flight.
  if (!grouped) return 1;
  return p.G % 2 == 0 ? 2 : 1;
}

cudaError_t launch_decode(const Problem& p, const void* q, const void* Kc, const void* Vc,
                          const Selection& sel, int num_splits, float* part_ml, float* part_acc,
                          void* O, float* LSE, cudaStream_t st, const KvLayout& kv, bool grouped) {
  if (p.bs != kBS) return cudaErrorNotSupported;
#define GBS_DEC(T, DD) \
  return decode_heads<T, DD>(p, q, Kc, Vc, sel, kv, grouped, num_splits, part_ml, part_acc, O, LSE, st)
  if (p.dtype == GBS_F32) {
    if (p.d == 64) GBS_DEC(float, 64);
    if (p.d == 128) GBS_DEC(float, 128);
  } else {
    if (p.d == 64) GBS_DEC(__nv_bfloat16, 64);
    if (p.d == 128) GBS_DEC(__nv_bfloat16, 128);
  }
#undef GBS_DEC
  return cudaErrorNotSupported;
}

}  // namespace gbs
