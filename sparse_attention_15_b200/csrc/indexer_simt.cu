// Lightning-indexer scores on the CUDA cores (float32 FMA).
//
// [AXK2] "SK Telecom 三大改进 / 1. Sparse Gated Attention（SGA）":
//   index_score[b,s,t] = sum_h weight[b,s,h] * softmax_scale * (q[b,s,h,:] . k[b,t,:]),
// with the causal mask imposed while scoring (-inf for keys after the query).
//
// This kernel serves the float32 workloads and any bf16 shape the tensor-core kernel
// does not take.  Tile: 128 keys x 8 queries per CTA; warp w owns query s0+w, lane l owns
// keys t0+l+32j (j<4).  The key tile is staged in shared memory as float32 with a padded
// row stride (conflict-free 16-byte reads); the warp-uniform query row is read straight
// from global memory (broadcast).
#include "common.cuh"
#include "kernels.h"

namespace dsa {

namespace {

constexpr int kKeys = 128;
constexpr int kQueries = 8;

template <typename T, int RELU>
__global__ void __launch_bounds__(256) index_scores_simt_kernel(
    const T* __restrict__ q_idx, const T* __restrict__ k_idx, const float* __restrict__ w,
    float scale, int S, int Tn, int HI, int DI, int q_off, float* __restrict__ scores) {
  extern __shared__ float4 smem_f4[];
  float* ks = reinterpret_cast<float*>(smem_f4);
  const int ld = DI + 4;
  const int b = blockIdx.z;
  const int t0 = blockIdx.x * kKeys;
  const int s0 = blockIdx.y * kQueries;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int s = s0 + warp;
  const float ninf = __int_as_float(0xff800000);

  const int s_hi = min(s0 + kQueries, S) - 1;  // last query of the tile
  if (t0 > s_hi + q_off) {
    // tile entirely in the future of every query: all -inf
    if (s < S) {
      float* row = scores + ((size_t)b * S + s) * Tn;
      for (int j = 0; j < 4; ++j) {
        int t = t0 + lane + 32 * j;
        if (t < Tn) row[t] = ninf;
      }
    }
    return;
  }

  // stage the key tile (float32)
  const T* kb = k_idx + ((size_t)b * Tn) * DI;
  for (int e = threadIdx.x * 4; e < kKeys * DI; e += blockDim.x * 4) {
    int r = e / DI, d = e % DI;
    int t = t0 + r;
    float x[4] = {0.f, 0.f, 0.f, 0.f};
    if (t < Tn) load4(kb + (size_t)t * DI + d, x);
    *reinterpret_cast<float4*>(ks + r * ld + d) = make_float4(x[0], x[1], x[2], x[3]);
  }
  __syncthreads();
  if (s >= S) return;

  const T* qrow = q_idx + (((size_t)b * S + s) * HI) * DI;
  const float* wrow = w + ((size_t)b * S + s) * HI;
  float tot[4] = {0.f, 0.f, 0.f, 0.f};
  for (int h = 0; h < HI; ++h) {
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    const T* qh = qrow + (size_t)h * DI;
    for (int d = 0; d < DI; d += 4) {
      float qv[4];
      load4(qh + d, qv);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float4 kv = *reinterpret_cast<const float4*>(ks + (lane + 32 * j) * ld + d);
        acc[j] = fmaf(qv[0], kv.x, acc[j]);
        acc[j] = fmaf(qv[1], kv.y, acc[j]);
        acc[j] = fmaf(qv[2], kv.z, acc[j]);
        acc[j] = fmaf(qv[3], kv.w, acc[j]);
      }
    }
    const float wh = wrow[h];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float a = RELU == 2 ? fmaxf(acc[j], 0.f) : acc[j];
      tot[j] = fmaf(wh, a, tot[j]);
    }
  }
  float* row = scores + ((size_t)b * S + s) * Tn;
  const int spos = s + q_off;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    int t = t0 + lane + 32 * j;
    if (t >= Tn) continue;
    float v = tot[j] * scale;
    if (RELU == 1) v = fmaxf(v, 0.f);
    row[t] = (t <= spos) ? v : ninf;
  }
}

template <typename T>
cudaError_t launch_typed(const void* q_idx, const void* k_idx, const float* w, float scale,
                         int relu, int B, int S, int T_, int HI, int DI, int q_off,
                         float* scores, cudaStream_t st) {
  dim3 grid((T_ + kKeys - 1) / kKeys, (S + kQueries - 1) / kQueries, B);
  size_t smem = (size_t)kKeys * (DI + 4) * sizeof(float);
  auto* qi = static_cast<const T*>(q_idx);
  auto* ki = static_cast<const T*>(k_idx);
  void (*kern)(const T*, const T*, const float*, float, int, int, int, int, int, float*) =
      relu == 1 ? index_scores_simt_kernel<T, 1>
                : (relu == 2 ? index_scores_simt_kernel<T, 2> : index_scores_simt_kernel<T, 0>);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<grid, 256, smem, st>>>(qi, ki, w, scale, S, T_, HI, DI, q_off, scores);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_index_scores_simt(int dtype, const void* q_idx, const void* k_idx,
                                     const float* w, float scale, int relu, int B, int S,
                                     int T, int HI, int DI, int q_off, float* scores,
                                     cudaStream_t st) {
  if (dtype == 0)
    return launch_typed<float>(q_idx, k_idx, w, scale, relu, B, S, T, HI, DI, q_off, scores,
                               st);
  return launch_typed<__nv_bfloat16>(q_idx, k_idx, w, scale, relu, B, S, T, HI, DI, q_off,
                                     scores, st);
}

}  // namespace dsa
