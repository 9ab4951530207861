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
// name is only a host-side stand-in, so its device address is looked up once per device with
// cudaGetSymbolAddress (on the first call made with that device current) and passed to the
// kernels.  Every GPU that loads the library holds the array until the process exits.
#include <stdio.h>

#include <mutex>

#include "../../include/dsa.h"
#include "common.cuh"
#include "kernels.h"

namespace {

constexpr size_t kNoAllocScratchBytes = 16u << 20;  // 16 MiB per device
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mu;

// Device address of g_noalloc_scratch on the current device (looked up once per device).
cudaError_t scratch_address(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

bool is_aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

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
  if (dtype != DSA_F32 && dtype != DSA_BF16)
    return reject(DSA_ERR_INVALID_ARG, "dsa_sparse_attn_noalloc: unknown dtype");
  if (!q || !k || !v || !idx || !out)
    return reject(DSA_ERR_INVALID_ARG, "dsa_sparse_attn_noalloc: null pointer argument");
  if (B <= 0 || S <= 0 || T <= 0 || H <= 0 || DQK <= 0 || DV <= 0 || K <= 0 || T < S)
    return reject(DSA_ERR_INVALID_ARG, "dsa_sparse_attn_noalloc: invalid sizes");
  if (gate_mode < DSA_GATE_OFF || gate_mode > DSA_GATE_SILU ||
      (gate_mode == DSA_GATE_OFF) != (gate == nullptr))
    return reject(DSA_ERR_INVALID_ARG, "dsa_sparse_attn_noalloc: invalid gate arguments");
  if (sm_scale != sm_scale || sm_scale > 3.0e38f || sm_scale < -3.0e38f)
    return reject(DSA_ERR_INVALID_ARG, "dsa_sparse_attn_noalloc: sm_scale not finite");
  const int vec = dtype == DSA_F32 ? 4 : 8;
  const size_t es = dtype == DSA_F32 ? 4 : 2;
  if (DQK > 256 || DV > 256 || DQK % vec || DV % vec || H > 64 || (H * DQK * es) % 16 ||
      (H * DV * es) % 16)
    return reject(DSA_ERR_UNSUPPORTED, "dsa_sparse_attn_noalloc: unsupported head shape");
  if (!is_aligned16(q) || !is_aligned16(k) || !is_aligned16(v) || !is_aligned16(idx) ||
      !is_aligned16(out) || (gate && !is_aligned16(gate)))
    return reject(DSA_ERR_UNSUPPORTED, "dsa_sparse_attn_noalloc: pointers must be 16-byte aligned");
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
