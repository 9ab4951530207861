// The indexer's Hadamard rotation of its inputs.
//
// [AXK2] SGA notes: the upstream indexer rotates q_I and k_I with a Hadamard transform
// (rotate_activation) before quantising them for its FP8 scoring kernel; the transform is
// orthogonal, so (Hq) . (Hk) = q . k and the scores are unchanged while the values are
// spread evenly over the dimensions (what the quantiser needs).
//
// out[r, :] = x[r, :] @ H / sqrt(d), H the d x d Sylvester Hadamard matrix (natural order),
// d in {64, 128}: the fast Walsh-Hadamard butterfly.  A warp takes kRows rows, with every
// row's loads issued before the first butterfly (memory-level parallelism); lane l holds
// the E = d/32 consecutive elements l*E .. l*E+E-1 of each.  The butterfly of stride h
// pairs elements k and k + h (bit h of k clear) into (a + b, a - b): strides below E stay
// inside a lane, stride E*m is the lane pair (l, l ^ m), exchanged with one shuffle per
// element.  Float32 arithmetic, one rounding to the output type.  In place is allowed
// (out == x): a warp reads its rows before writing them.
#include "common.cuh"
#include "kernels.h"

namespace dsa {

namespace {

constexpr int kRows = 4;  // rows per warp

template <typename T, int D>
__global__ void hadamard_kernel(const T* __restrict__ x, T* __restrict__ out, long long rows) {
  constexpr int E = D / 32;
  static_assert(E == 2 || E == 4, "d must be 64 or 128");
  const long long warp_id = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const long long row0 = warp_id * kRows;
  const int lane = threadIdx.x & 31;
  if (row0 >= rows) return;
  float v[kRows][E];
#pragma unroll
  for (int r = 0; r < kRows; ++r) {
    const T* src = x + (row0 + r) * D + lane * E;
#pragma unroll
    for (int i = 0; i < E; ++i) v[r][i] = row0 + r < rows ? to_f32(src[i]) : 0.f;
  }
#pragma unroll
  for (int r = 0; r < kRows; ++r) {
    // strides 1 (and 2) inside the lane
#pragma unroll
    for (int h = 1; h < E; h <<= 1)
#pragma unroll
      for (int i = 0; i < E; ++i)
        if (!(i & h)) {
          const float a = v[r][i], b = v[r][i + h];
          v[r][i] = a + b;
          v[r][i + h] = a - b;
        }
    // strides E, 2E, ..., 16E across lanes
#pragma unroll
    for (int m = 1; m < 32; m <<= 1) {
      const bool upper = lane & m;  // this lane holds the k + h halves of its pairs
#pragma unroll
      for (int i = 0; i < E; ++i) {
        const float p = __shfl_xor_sync(0xffffffffu, v[r][i], m);
        v[r][i] = upper ? p - v[r][i] : v[r][i] + p;
      }
    }
  }
  const float scale = D == 64 ? 0.125f : 0.08838834764831845f;  // 1/sqrt(d)
#pragma unroll
  for (int r = 0; r < kRows; ++r) {
    if (row0 + r >= rows) break;
    T* dst = out + (row0 + r) * D + lane * E;
#pragma unroll
    for (int i = 0; i < E; ++i) dst[i] = from_f32<T>(v[r][i] * scale);
  }
}

template <typename T>
cudaError_t launch_t(const void* x, void* out, long long rows, int d, cudaStream_t st) {
  const long long per_cta = 8LL * kRows;  // 8 warps per CTA
  const unsigned grid = (unsigned)((rows + per_cta - 1) / per_cta);
  if (d == 128)
    hadamard_kernel<T, 128><<<grid, 256, 0, st>>>(static_cast<const T*>(x), static_cast<T*>(out),
                                                  rows);
  else
    hadamard_kernel<T, 64><<<grid, 256, 0, st>>>(static_cast<const T*>(x), static_cast<T*>(out),
                                                 rows);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_hadamard(int dtype, const void* x, void* out, long long rows, int d,
                            cudaStream_t st) {
  if (rows <= 0) return cudaSuccess;
  if (d != 64 && d != 128) return cudaErrorNotSupported;
  if (rows > (long long)8 * 0x7fffffff) return cudaErrorInvalidValue;
  return dtype == 0 ? launch_t<float>(x, out, rows, d, st)
                    : launch_t<__nv_bfloat16>(x, out, rows, d, st);
}

}  // namespace dsa
