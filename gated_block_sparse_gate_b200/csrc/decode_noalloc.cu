// decode_noalloc.cu — gbs_decode_noalloc: the sparse decode for callers that
// cannot hand the library a workspace.
//
// gbs_decode needs a caller-allocated workspace for the Top-K lists and the
// per-split partial results. Some callers cannot allocate device memory at the
// point where they decode: a serving loop whose device memory is entirely
// reserved up front by another allocator, or one that must never call
// cudaMalloc on its hot path because that call can synchronise the device and
// stall every other stream. This variant keeps that scratch in one statically
// sized device array that lives in the library itself, so the caller only
// passes inputs and outputs.
//
// The array is a file-scope __device__ object: every GPU that loads the
// library holds GBS_DECODE_NOALLOC_SCRATCH_BYTES of it until the process exits.
// Host code cannot use the array's name as a device address, so the first call
// on each device looks the address up once with cudaGetSymbolAddress (with
// that device current) and caches it; make that first call before any stream
// capture. All calls on a device share the one array and it keeps the last
// call's contents; nothing in it needs to start at zero because every call
// rewrites what it reads. Calls that overlap on the GPU (different streams, or
// host threads racing) overwrite each other's scratch and must be serialised
// by the caller.
#include <mutex>
#include <stdio.h>

#include "common.cuh"
#include "internal.h"

namespace {

constexpr size_t kScratchBytes = GBS_DECODE_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_decode_scratch[kScratchBytes];

std::mutex g_setup_mutex;
void* g_scratch_addr[kMaxDevices] = {};

gbs_status noalloc_fail(gbs_status s, const char* msg) {
  char buf[256];
  snprintf(buf, sizeof(buf), "gbs_decode_noalloc: %s", msg);
  gbs::set_last_error(buf);
  return s;
}

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

// Bytes of scratch a call with these sizes uses.
size_t scratch_needed(size_t rows, int topk, int splits, int d) {
  return align256(rows * topk * sizeof(int32_t)) + align256(rows * sizeof(int32_t)) +
         align256(rows * topk * sizeof(float)) + align256(rows * splits * 2 * sizeof(float)) +
         align256(rows * splits * d * sizeof(float));
}

// Device address of the scratch array on the current device (looked up once).
gbs_status scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return noalloc_fail(GBS_ERR_CUDA, cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return noalloc_fail(GBS_ERR_UNSUPPORTED, "device index too large");
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (!g_scratch_addr[dev]) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_decode_scratch);
    if (e != cudaSuccess || !ptr) return noalloc_fail(GBS_ERR_CUDA, "cudaGetSymbolAddress failed");
    g_scratch_addr[dev] = ptr;
  }
  *out = g_scratch_addr[dev];
  return GBS_OK;
}

}  // namespace

extern "C" gbs_status gbs_decode_noalloc(const gbs_params* in, const void* q, const void* Kc,
                                         const void* Vc, const float* S, void* O, float* LSE,
                                         int num_splits, void* stream) {
  gbs::set_last_error("");
  // the same validation as gbs_decode (shape, mode, dtype, size limits)
  gbs::Problem pr{};
  gbs_status s = gbs::resolve_params(in, GBS_OP_DECODE, &pr);
  if (s != GBS_OK) return s;
  if (num_splits < 0 || num_splits > gbs::kMaxDecodeSplits)
    return noalloc_fail(GBS_ERR_INVALID_ARG, "num_splits must be in [0, 32]");
  const void* ptrs[] = {q, Kc, Vc, S, O, LSE};
  for (const void* ptr : ptrs)
    if (!ptr || ((uintptr_t)ptr & 15u))
      return noalloc_fail(GBS_ERR_INVALID_ARG, "a tensor pointer is NULL or not 16-byte aligned");

  const size_t rows = (size_t)pr.B * pr.Hq;
  const int cur = (pr.N - 1) / pr.bs;
  const int n_ent = (pr.topk < cur ? pr.topk : cur) + 1;
  int splits = num_splits;
  if (splits == 0) {
    // gbs_decode's rule, stepped down only if its partials would not fit
    cudaError_t e = gbs::decode_auto_splits(pr, false, n_ent, &splits);
    if (e != cudaSuccess) return noalloc_fail(GBS_ERR_CUDA, cudaGetErrorString(e));
    while (splits > 1 && scratch_needed(rows, pr.topk, splits, pr.d) > kScratchBytes) --splits;
  }
  if (splits > n_ent) splits = n_ent;
  if (splits < 1) splits = 1;
  if (scratch_needed(rows, pr.topk, splits, pr.d) > kScratchBytes)
    return noalloc_fail(GBS_ERR_INVALID_ARG,
                        "B*Hq, topk, splits and d need more than the static scratch "
                        "(GBS_DECODE_NOALLOC_SCRATCH_BYTES); use gbs_decode with a workspace");

  void* base = nullptr;
  s = scratch_address(&base);
  if (s != GBS_OK) return s;
  char* c = static_cast<char*>(base);
  gbs::Selection sel{};
  sel.idx = reinterpret_cast<int32_t*>(c);
  c += align256(rows * pr.topk * sizeof(int32_t));
  sel.cnt = reinterpret_cast<int32_t*>(c);
  c += align256(rows * sizeof(int32_t));
  sel.logg = reinterpret_cast<float*>(c);
  c += align256(rows * pr.topk * sizeof(float));
  float* part_ml = reinterpret_cast<float*>(c);
  c += align256(rows * splits * 2 * sizeof(float));
  float* part_acc = reinterpret_cast<float*>(c);

  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e = gbs::launch_select(S, (int)rows, pr.Nb, 1, cur, pr.topk, pr.mode, pr.log_tau,
                                     sel.idx, sel.cnt, sel.logg, nullptr, st);
  if (e == cudaSuccess)
    e = gbs::launch_decode(pr, q, Kc, Vc, sel, splits, part_ml, part_acc, O, LSE, st,
                           gbs::KvLayout(), false);
  if (e != cudaSuccess) return noalloc_fail(GBS_ERR_CUDA, cudaGetErrorString(e));
  return GBS_OK;
}
