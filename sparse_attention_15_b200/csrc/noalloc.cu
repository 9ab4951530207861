// dsa_sparse_attn_noalloc: the gather form of dsa_sparse_attn for callers that cannot
// allocate device memory.
//
// Some callers only ever receive the input and output buffers and may not create device
// memory of their own: a plugin inside an inference runtime whose memory planner owns every
// device byte, or a decode loop with a fixed memory budget that must not pay for the
// implicit synchronisation and fragmentation of a fresh allocation.  dsa_sparse_attn needs a
// caller-provided workspace for its split-key partial results; this entry point keeps those
// partials in a fixed array in the library's own device memory instead, so the caller passes
// inputs and outputs only and nothing is allocated on any call.
//
// The array is a file-scope __device__ variable of kNoAllocScratchBytes.  In host code its
// name is only a host-side stand-in, so its device address is looked up with
// cudaGetSymbolAddress once per CUDA context (on the first call made in that context, the
// current device's) and passed to the kernels.  The cache is keyed by the context's
// process-unique ID, so a context created later on the same device -- after
// cudaDeviceReset, or a driver-API context made current by the caller -- gets a fresh
// lookup instead of a stale address.  Every GPU that loads the library holds the array
// until the process exits.
#include <stdio.h>

#include <mutex>

#include "../../include/dsa.h"
#include "checks.h"
#include "common.cuh"
#include "kernels.h"

namespace {

constexpr size_t kNoAllocScratchBytes = 16u << 20;  // 16 MiB per device
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// (context ID, device address of g_noalloc_scratch in that context), most recent first.
struct ScratchEntry {
  unsigned long long ctx_id;
  void* addr;
};
constexpr int kMaxContexts = 16;
ScratchEntry g_scratch_cache[kMaxContexts] = {};
int g_scratch_entries = 0;
std::mutex g_scratch_mu;

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// The current context's process-unique ID; false if the driver does not provide it.
bool current_context_id(unsigned long long* id) {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  CUcontext ctx = nullptr;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}

// Device address of g_noalloc_scratch in the current context.  When no context is current
// yet, cudaGetSymbolAddress makes the current device's primary context current, and the
// entry is keyed by that context.
cudaError_t scratch_address(void** out) {
  cudaError_t e;
  unsigned long long id = 0;
  const bool have_id = current_context_id(&id);
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (have_id) {
    for (int i = 0; i < g_scratch_entries; ++i)
      if (g_scratch_cache[i].ctx_id == id) {
        *out = g_scratch_cache[i].addr;
        return cudaSuccess;
      }
  }
  void* p = nullptr;
  e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (e != cudaSuccess) return e;
  // the lookup may have made the primary context current: key the entry by that context
  if (!have_id && !current_context_id(&id)) {
    *out = p;  // no context IDs from this driver: look the address up on every call
    return cudaSuccess;
  }
  const int n = g_scratch_entries < kMaxContexts ? g_scratch_entries + 1 : kMaxContexts;
  for (int i = n - 1; i > 0; --i) g_scratch_cache[i] = g_scratch_cache[i - 1];
  g_scratch_cache[0] = ScratchEntry{id, p};
  g_scratch_entries = n;
  *out = p;
  return cudaSuccess;
}

dsa_status reject(dsa_status st, const char* msg) {
  dsa::set_last_error(msg);
  return st;
}

}  // namespace

extern "C" {

size_t dsa_sparse_attn_noalloc_max_scratch_bytes(void) { return kNoAllocScratchBytes; }

dsa_status dsa_sparse_attn_noalloc(dsa_dtype dtype, const void* q, const void* k, const void* v,
                                   const int32_t* idx, int K, const void* gate,
                                   dsa_gate_mode gate_mode, float sm_scale, int B, int S, int T,
                                   int H, int DQK, int DV, void* out, dsa_stream_t stream) {
  // the same argument checks as dsa_sparse_attn (same statuses and messages)
  dsa_status st = dsa::check_attn_common(dtype, q, k, v, gate, gate_mode, sm_scale, B, S, T, H,
                                         H, DQK, DV, out);
  if (st != DSA_OK) return st;
  if ((st = dsa::check_idx_args(idx, K)) != DSA_OK) return st;
  const size_t need = dsa::gather_attn_workspace_bytes(B, S, H, DV, K);
  if (need > kNoAllocScratchBytes) {
    char msg[256];
    snprintf(msg, sizeof(msg),
             "dsa_sparse_attn_noalloc: this shape needs %zu bytes of split-key scratch, more "
             "than the fixed %zu bytes; use dsa_sparse_attn with a workspace",
             need, kNoAllocScratchBytes);
    return reject(DSA_ERR_UNSUPPORTED, msg);
  }
  void* scratch = nullptr;
  if (need > 0) {
    const cudaError_t e = scratch_address(&scratch);
    if (e != cudaSuccess) {
      char msg[256];
      snprintf(msg, sizeof(msg), "dsa_sparse_attn_noalloc: scratch lookup failed: %s",
               cudaGetErrorString(e));
      return reject(DSA_ERR_CUDA, msg);
    }
  }
  dsa::AttnProblem p{};
  p.dtype = (int)dtype; p.q = q; p.k = k; p.v = v; p.idx = idx; p.K = K; p.window = 0;
  p.gate = gate; p.gate_mode = (int)gate_mode;
  p.sm_scale = sm_scale > 0.f ? sm_scale : 1.0f / sqrtf((float)DQK);
  p.B = B; p.S = S; p.T = T; p.H = H; p.HKV = H; p.DQK = DQK; p.DV = DV; p.q_off = T - S;
  p.out = out;
  const cudaError_t e =
      dsa::launch_gather_attn(p, scratch, kNoAllocScratchBytes, (cudaStream_t)stream);
  if (e == cudaErrorNotSupported)
    return reject(DSA_ERR_UNSUPPORTED, "dsa_sparse_attn_noalloc: no kernel for this shape");
  if (e != cudaSuccess) {
    char msg[256];
    snprintf(msg, sizeof(msg), "dsa_sparse_attn_noalloc: %s", cudaGetErrorString(e));
    return reject(DSA_ERR_CUDA, msg);
  }
  return DSA_OK;
}

}  // extern "C"
