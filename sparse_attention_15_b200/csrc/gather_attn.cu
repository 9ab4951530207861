// Sparse attention by gathering the selected K/V rows, with the headwise gate fused.
//
// [AXK2] "注意力前向的骨架：MLA + 显式稀疏掩码": every query attends only to the keys the
// indexer selected (all other positions are -inf), under the causal mask; the cache holds
// the expanded per-head K/V (the expand_kv output).  [DSV2] items 4-6: q/k heads are
// qk_nope + qk_rope wide, v heads v_head_dim wide.  [SPARK] "前向流程": the output of
// head h is multiplied by act(gate[b,s,h]) in float32 before the cast.
//
// All heads of a query share its index set, so one selected key is one contiguous row of
// the K cache (H*DQK elements) and one of the V cache (H*DV elements).  A producer warp
// streams those rows into a ring of shared-memory slots with 1-D bulk copies (the TMA
// engine, mbarrier transaction counts, no multicast); consumer warps own whole heads
// (lane l holds dims 4l..4l+3 of every 128-wide slice) and run an online softmax in
// float32, one key at a time, without any block-wide barrier.  Each consumer warp releases
// a slot by arriving on its "empty" barrier.
//
// The same kernel computes the sliding-window layers: the index set is then the band
// s+q_off-window < t <= s+q_off, and query head h reads KV head h / (H / HKV).
//
// Long index lists with few query rows (decode) are split over several CTAs; each writes
// an unnormalised partial (o, m, l) and a second kernel merges them in a fixed order.
#include <atomic>

#include "common.cuh"
#include "kernels.h"

namespace dsa {

namespace {

// Testing aid (dsa_test_arm_wait_timeout): when armed, the next gather launch's first CTA
// fills none of its slots, so that CTA's consumers wait on a slot that never fills until
// their bounded wait runs out and records the timeout.  One-shot.
std::atomic<int> g_arm_skip_copy{0};

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLazyRescale = 8.0f;  // raise the running max only past 2^8 (log2 units)

// Warp sums of N per-lane partials (N = 1, 2, 4), every lane receiving all N sums.  The
// first butterfly steps halve the values each lane carries (lanes split the heads between
// them), so N sums cost N + 4 shuffles (plus N broadcasts) instead of 5N.
template <int N>
__device__ __forceinline__ void warp_sum_heads(const float (&x)[N], float (&out)[N]) {
  const int lane = threadIdx.x & 31;
  if constexpr (N == 1) {
    float v = x[0];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    out[0] = v;
  } else if constexpr (N == 2) {
    const bool up = lane & 16;  // lanes 16..31 keep head 1
    const float send = up ? x[0] : x[1];
    const float keep = up ? x[1] : x[0];
    float v = keep + __shfl_xor_sync(0xffffffffu, send, 16);
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    out[0] = __shfl_sync(0xffffffffu, v, 0);
    out[1] = __shfl_sync(0xffffffffu, v, 16);
  } else {
    static_assert(N == 4, "1, 2 or 4 heads per warp");
    const bool up16 = lane & 16, up8 = lane & 8;
    // step 1: lanes 16..31 keep heads 2,3; lanes 0..15 keep heads 0,1
    const float s0 = up16 ? x[0] : x[2], s1 = up16 ? x[1] : x[3];
    const float k0 = up16 ? x[2] : x[0], k1 = up16 ? x[3] : x[1];
    const float a0 = k0 + __shfl_xor_sync(0xffffffffu, s0, 16);
    const float a1 = k1 + __shfl_xor_sync(0xffffffffu, s1, 16);
    // step 2: within each half, lanes with bit 3 set keep the second head of the pair
    float v = (up8 ? a1 : a0) + __shfl_xor_sync(0xffffffffu, up8 ? a0 : a1, 8);
#pragma unroll
    for (int o = 4; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    // lane 0: head 0, lane 8: head 1, lane 16: head 2, lane 24: head 3
#pragma unroll
    for (int i = 0; i < 4; ++i) out[i] = __shfl_sync(0xffffffffu, v, 8 * i);
  }
}

struct GatherArgs {
  const void* q;
  const void* k;
  const void* v;
  const int32_t* idx;
  const void* gate;
  void* out;
  float* part_o;   // [rows, nsplit, H, DV] (split mode)
  float* part_ml;  // [rows, nsplit, H, 2]
  int K, window, gate_mode;
  float qk_scale;  // sm_scale * log2(e)
  int S, T, H, HKV, DQK, DV, q_off;
  int nsplit, keys_per_split;
  int nslots;
  uint32_t k_bytes, v_bytes, slot_bytes;
  uint32_t key_list_bytes;  // shared-memory bytes reserved for the key list
  const void* sink_k;       // [nsink, HKV, DQK] attention sinks (PAS) or NULL
  const void* sink_v;       // [nsink, HKV, DV]
  int nsink;
  int skip_first_copy;      // testing aid: CTA 0 fills no slot
};

// Entry jj of a query's key list: with SINKS the nsink sinks come first (encoded as
// -2 - sink), then the selected keys (or the band).  -1 marks an entry to skip.
template <bool SINKS>
__device__ __forceinline__ int key_at(const GatherArgs& a, const int32_t* idx_row, int jj,
                                      int spos) {
  if (SINKS && jj < a.nsink) return -2 - jj;
  const int e = SINKS ? jj - a.nsink : jj;
  const int t = idx_row ? __ldg(idx_row + e) : spos - a.window + 1 + e;  // band: oldest first
  return (t >= 0 && t < a.T && t <= spos) ? t : -1;
}

// SINKS: the key lists start with attention sinks (a separate instantiation, so the common
// path carries none of their arithmetic).
template <typename T, int QKV, int VV, int HPW, bool SINKS>
__global__ void __launch_bounds__(544, HPW <= 2 ? 2 : 1) gather_attn_kernel(const GatherArgs a) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int nslots = a.nslots;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);
  uint64_t* empty = full + nslots;
  int* slot_key = reinterpret_cast<int*>(empty + nslots);
  int* keys = reinterpret_cast<int*>(smem + 1024);    // this CTA's key list
  uint8_t* slots = smem + 1024 + a.key_list_bytes;   // K/V row slots

  const int nw = (blockDim.x >> 5) - 1;  // consumer warps; the last warp produces
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x / a.nsplit;
  const int split = blockIdx.x % a.nsplit;
  const int b = row / a.S, s = row % a.S;
  const int spos = s + a.q_off;
  const int nkeys_total = (SINKS ? a.nsink : 0) + (a.idx ? a.K : a.window);
  const int j0 = split * a.keys_per_split;
  const int nkeys = max(0, min(nkeys_total, j0 + a.keys_per_split) - j0);
  const int32_t* idx_row = a.idx ? a.idx + (size_t)row * a.K : nullptr;

  if (threadIdx.x == 0) {
    for (int i = 0; i < nslots; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], nw);
    }
    fence_mbar_init();
  }
  __syncthreads();

  const T* kbase = static_cast<const T*>(a.k) + (size_t)b * a.T * a.HKV * a.DQK;
  const T* vbase = static_cast<const T*>(a.v) + (size_t)b * a.T * a.HKV * a.DV;

  if (warp == nw) {
    // ------------------------------------------------------------- producer
    // stage the key list once (coalesced), then issue the row copies back to back
    for (int j = lane; j < nkeys; j += 32)
      keys[j] = key_at<SINKS>(a, idx_row, j0 + j, spos);
    __syncwarp();
    if (lane == 0) {
      const bool skip_first = a.skip_first_copy != 0 && blockIdx.x == 0;
      int issued = 0;  // keys whose slot fill was issued
      for (int j = 0; j < nkeys; ++j) {
        const int slot = j % nslots;
        const int round = j / nslots;
        if (round > 0 && !mbar_wait(&empty[slot], (round - 1) & 1)) break;
        // testing aid: the first slot never fills and nothing more is issued, so this CTA
        // has no copy in flight while its consumers wait for that slot until they give up
        if (skip_first) break;
        issued = j + 1;
        const int t = keys[j];
        slot_key[slot] = t;
        if (SINKS ? t != -1 : t >= 0) {
          // a cache row, or (t <= -2) sink row -2 - t, which no batch row owns
          const T* ksrc = kbase + (size_t)t * a.HKV * a.DQK;
          const T* vsrc = vbase + (size_t)t * a.HKV * a.DV;
          if (SINKS && t < 0) {
            ksrc = static_cast<const T*>(a.sink_k) + (size_t)(-2 - t) * a.HKV * a.DQK;
            vsrc = static_cast<const T*>(a.sink_v) + (size_t)(-2 - t) * a.HKV * a.DV;
          }
          uint8_t* dst = slots + (size_t)slot * a.slot_bytes;
          mbar_arrive_expect_tx(&full[slot], a.k_bytes + a.v_bytes);
          bulk_g2s(dst, ksrc, a.k_bytes, &full[slot]);
          bulk_g2s(dst + a.k_bytes, vsrc, a.v_bytes, &full[slot]);
        } else {
          mbar_arrive(&full[slot]);
        }
      }
      // Copies still in flight must land before the CTA exits, also when the consumers gave
      // up early (a recorded timeout): wait, bounded, for the last fill of every slot that
      // had a copy issued.
      for (int j = issued - 1; j >= 0 && j >= issued - nslots; --j) {
        const int t = keys[j];
        if (SINKS ? t != -1 : t >= 0) drain_wait(&full[j % nslots], (j / nslots) & 1);
      }
    }
    return;
  }

  // --------------------------------------------------------------- consumers
  // Per key and head: dot = q.k (lanes hold 4 dims of each 128-wide slice), one butterfly
  // reduction for every pair of heads, p = 2^(dot - m), acc += p v.  The running max m is
  // only raised when a key exceeds it by more than 2^8 (p <= 256 otherwise), so the
  // accumulator is rescaled rarely rather than on every key; the final (acc, m, l) is the
  // same softmax as with a strict running max.
  constexpr int hpw = HPW;  // heads per warp
  const int group = a.H / a.HKV;
  float qr[hpw][QKV][4];
  float acc[hpw][VV][4];
  float m[hpw], l[hpw];
  int koff[hpw], voff[hpw];  // element offsets of this warp's heads inside a slot
  const T* qrow = static_cast<const T*>(a.q) + (size_t)row * a.H * a.DQK;
#pragma unroll
  for (int hi = 0; hi < hpw; ++hi) {
    const int h = warp + nw * hi;
    const int kvh = h / group;
    koff[hi] = kvh * a.DQK;
    voff[hi] = kvh * a.DV;
    m[hi] = -INFINITY;
    l[hi] = 0.f;
#pragma unroll
    for (int c = 0; c < VV; ++c)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[hi][c][e] = 0.f;
#pragma unroll
    for (int c = 0; c < QKV; ++c) {
      const int d = c * 128 + lane * 4;
      float x[4] = {0.f, 0.f, 0.f, 0.f};
      if (d < a.DQK) load4(qrow + (size_t)h * a.DQK + d, x);
#pragma unroll
      for (int e = 0; e < 4; ++e) qr[hi][c][e] = x[e] * a.qk_scale;
    }
  }

  bool ok = true;
  int slot = 0;
  uint32_t phase = 0;
  for (int j = 0; j < nkeys && ok; ++j) {
    ok = warp_wait(&full[slot], phase);  // warp-uniform: the shuffles below need all lanes
    if (ok && (SINKS ? slot_key[slot] != -1 : slot_key[slot] >= 0)) {
      const T* ks = reinterpret_cast<const T*>(slots + (size_t)slot * a.slot_bytes);
      const T* vs = reinterpret_cast<const T*>(slots + (size_t)slot * a.slot_bytes + a.k_bytes);
      float part[hpw];
#pragma unroll
      for (int hi = 0; hi < hpw; ++hi) {
        float dot = 0.f;
#pragma unroll
        for (int c = 0; c < QKV; ++c) {
          const int d = c * 128 + lane * 4;
          if (d < a.DQK) {
            float x[4];
            load4(ks + koff[hi] + d, x);
#pragma unroll
            for (int e = 0; e < 4; ++e) dot = fmaf(qr[hi][c][e], x[e], dot);
          }
        }
        part[hi] = dot;
      }
      float dots[hpw];
      warp_sum_heads<hpw>(part, dots);
#pragma unroll
      for (int hi = 0; hi < hpw; ++hi) {
        const float dot = dots[hi];
        if (dot > m[hi] + kLazyRescale) {  // warp-uniform: every lane holds the same dot
          const float alpha = ex2_ftz(m[hi] - dot);  // 0 for the first key (m = -inf)
          l[hi] *= alpha;
#pragma unroll
          for (int c = 0; c < VV; ++c)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[hi][c][e] *= alpha;
          m[hi] = dot;
        }
        const float p = ex2_ftz(dot - m[hi]);
        l[hi] += p;
#pragma unroll
        for (int c = 0; c < VV; ++c) {
          const int d = c * 128 + lane * 4;
          if (d < a.DV) {
            float x[4];
            load4(vs + voff[hi] + d, x);
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[hi][c][e] = fmaf(p, x[e], acc[hi][c][e]);
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[slot]);
    if (++slot == nslots) {
      slot = 0;
      phase ^= 1u;
    }
  }

  // --------------------------------------------------------------- epilogue
#pragma unroll
  for (int hi = 0; hi < hpw; ++hi) {
    const int h = warp + nw * hi;
    if (a.nsplit == 1) {
      float f = l[hi] > 0.f ? 1.0f / l[hi] : 0.f;
      if (a.gate)
        f *= gate_act(to_f32(static_cast<const T*>(a.gate)[(size_t)row * a.H + h]), a.gate_mode);
      T* o = static_cast<T*>(a.out) + ((size_t)row * a.H + h) * a.DV;
#pragma unroll
      for (int c = 0; c < VV; ++c) {
        const int d = c * 128 + lane * 4;
        if (d < a.DV)
#pragma unroll
          for (int e = 0; e < 4; ++e) o[d + e] = from_f32<T>(acc[hi][c][e] * f);
      }
    } else {
      const size_t base = ((size_t)row * a.nsplit + split) * a.H + h;
      float* po = a.part_o + base * a.DV;
#pragma unroll
      for (int c = 0; c < VV; ++c) {
        const int d = c * 128 + lane * 4;
        if (d < a.DV)
          *reinterpret_cast<float4*>(po + d) =
              make_float4(acc[hi][c][0], acc[hi][c][1], acc[hi][c][2], acc[hi][c][3]);
      }
      if (lane == 0) {
        a.part_ml[base * 2 + 0] = m[hi];
        a.part_ml[base * 2 + 1] = l[hi];
      }
    }
  }
}

// Merge the split partials of one (row, head): out = sum_p 2^(m_p - M) o_p / sum_p 2^(m_p - M) l_p,
// summed in split order (deterministic).  One CTA per (row, head): the per-split weights are
// computed once into shared memory, then each thread combines one output element.
template <typename T>
__global__ void combine_kernel(const GatherArgs a) {
  __shared__ float wsplit[64];
  __shared__ float inv_l;
  const int row = blockIdx.x / a.H, h = blockIdx.x % a.H;
  const size_t base0 = (size_t)row * a.nsplit * a.H + h;  // partial (row, split 0, h)
  if (threadIdx.x < 32) {
    float M = -INFINITY;
    for (int p = threadIdx.x; p < a.nsplit; p += 32)
      M = fmaxf(M, a.part_ml[(base0 + (size_t)p * a.H) * 2]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    for (int p = threadIdx.x; p < a.nsplit; p += 32) {
      const float mp = a.part_ml[(base0 + (size_t)p * a.H) * 2];
      wsplit[p] = (M == -INFINITY || mp == -INFINITY) ? 0.f : exp2f(mp - M);
    }
    __syncwarp();
    if (threadIdx.x == 0) {
      float L = 0.f;
      for (int p = 0; p < a.nsplit; ++p)
        L = fmaf(a.part_ml[(base0 + (size_t)p * a.H) * 2 + 1], wsplit[p], L);
      float f = L > 0.f ? 1.0f / L : 0.f;
      if (a.gate)
        f *= gate_act(to_f32(static_cast<const T*>(a.gate)[(size_t)row * a.H + h]), a.gate_mode);
      inv_l = f;
    }
  }
  __syncthreads();
  for (int d = threadIdx.x; d < a.DV; d += blockDim.x) {
    float O = 0.f;
    for (int p = 0; p < a.nsplit; ++p)
      O = fmaf(a.part_o[(base0 + (size_t)p * a.H) * a.DV + d], wsplit[p], O);
    static_cast<T*>(a.out)[((size_t)row * a.H + h) * a.DV + d] = from_f32<T>(O * inv_l);
  }
}

// Heads per consumer warp: the smallest of 1, 2, 4 that divides H and leaves at most
// 16 consumer warps.
int heads_per_warp(int H) {
  for (int hpw = 1; hpw <= 4; hpw *= 2)
    if (H % hpw == 0 && H / hpw <= 16) return hpw;
  return 0;
}

// Split policy: few query rows and long key lists -> spread the keys over CTAs.  The split
// count is chosen so that rows * nsplit fills whole waves of the resident CTAs (two per SM
// on a 148-SM B200) as closely as possible, with at least 64 keys per split and at most 32
// splits; the fewest splits within 5% of full waves win.  Depends on the shape only (no
// device query), so workspace sizes are reproducible.
void split_policy(int rows, int nkeys, int* nsplit, int* kps, bool allow_split = true) {
  const int resident = 2 * 148;
  if (!allow_split || rows >= resident || nkeys <= 128) {
    *nsplit = 1;
    *kps = nkeys;
    return;
  }
  int max_ns = (nkeys + 63) / 64;
  if (max_ns > 32) max_ns = 32;
  // the fewest splits whose waves are at least 95% full; else the fullest
  int best = 1;
  double best_eff = -1.0;
  for (int ns = 1; ns <= max_ns; ++ns) {
    const int k = (nkeys + ns - 1) / ns;
    const int n = (nkeys + k - 1) / k;           // splits actually used
    const long long items = (long long)rows * n;
    const long long waves = (items + resident - 1) / resident;
    const double eff = (double)items / (double)(waves * resident);
    if (eff >= 0.95) {
      best = ns;
      break;
    }
    if (eff > best_eff + 1e-9) {
      best_eff = eff;
      best = ns;
    }
  }
  *kps = (nkeys + best - 1) / best;
  *nsplit = (nkeys + *kps - 1) / *kps;
}

template <typename T, int QKV, int VV, int HPW>
cudaError_t launch_t(GatherArgs a, int nw, size_t smem, unsigned grid, int rows,
                     cudaStream_t st) {
  auto kern = a.nsink > 0 ? gather_attn_kernel<T, QKV, VV, HPW, true>
                          : gather_attn_kernel<T, QKV, VV, HPW, false>;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<grid, 32 * (nw + 1), smem, st>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess || a.nsplit == 1) return e;
  combine_kernel<T><<<(unsigned)rows * a.H, 128, 0, st>>>(a);
  return cudaGetLastError();
}

template <typename T, int HPW>
cudaError_t launch_dims(GatherArgs a, int nw, size_t smem, unsigned grid, int rows,
                        cudaStream_t st) {
  const int qkv = (a.DQK + 127) / 128, vv = (a.DV + 127) / 128;
  if (qkv == 1 && vv == 1) return launch_t<T, 1, 1, HPW>(a, nw, smem, grid, rows, st);
  if (qkv == 2 && vv == 1) return launch_t<T, 2, 1, HPW>(a, nw, smem, grid, rows, st);
  if (qkv == 2 && vv == 2) return launch_t<T, 2, 2, HPW>(a, nw, smem, grid, rows, st);
  if (qkv == 1 && vv == 2) return launch_t<T, 1, 2, HPW>(a, nw, smem, grid, rows, st);
  return cudaErrorNotSupported;
}

template <typename T>
cudaError_t launch_hpw(GatherArgs a, int hpw, size_t smem, unsigned grid, int rows,
                       cudaStream_t st) {
  const int nw = a.H / hpw;
  if (hpw == 1) return launch_dims<T, 1>(a, nw, smem, grid, rows, st);
  if (hpw == 2) return launch_dims<T, 2>(a, nw, smem, grid, rows, st);
  if (hpw == 4) return launch_dims<T, 4>(a, nw, smem, grid, rows, st);
  return cudaErrorNotSupported;
}

}  // namespace

void arm_gather_skip_copy() { g_arm_skip_copy.store(1); }

cudaError_t launch_split_combine(int dtype, const float* part_o, const float* part_ml, int rows,
                                 int nsplit, int H, int DV, const void* gate, int gate_mode,
                                 void* out, cudaStream_t st) {
  if (rows <= 0) return cudaSuccess;
  if (nsplit < 1 || nsplit > 64) return cudaErrorInvalidValue;
  GatherArgs a{};
  a.part_o = const_cast<float*>(part_o);
  a.part_ml = const_cast<float*>(part_ml);
  a.nsplit = nsplit; a.H = H; a.DV = DV;
  a.gate = gate; a.gate_mode = gate_mode; a.out = out;
  const unsigned grid = (unsigned)rows * (unsigned)H;
  if (dtype == 0)
    combine_kernel<float><<<grid, 128, 0, st>>>(a);
  else
    combine_kernel<__nv_bfloat16><<<grid, 128, 0, st>>>(a);
  return cudaGetLastError();
}

size_t gather_attn_workspace_bytes(int B, int S, int H, int DV, int K, int nsink) {
  const int rows = B * S;
  int ns, kps;
  split_policy(rows, K + nsink, &ns, &kps);
  if (ns == 1) return 0;
  return (size_t)rows * ns * H * (DV + 2) * sizeof(float);
}

cudaError_t launch_gather_attn(const AttnProblem& p, void* ws, size_t ws_bytes,
                               cudaStream_t st) {
  GatherArgs a{};
  a.q = p.q; a.k = p.k; a.v = p.v; a.idx = p.idx; a.gate = p.gate; a.out = p.out;
  a.K = p.K; a.window = p.window; a.gate_mode = p.gate_mode;
  a.qk_scale = p.sm_scale * kLog2e;
  a.S = p.S; a.T = p.T; a.H = p.H; a.HKV = p.HKV; a.DQK = p.DQK; a.DV = p.DV; a.q_off = p.q_off;
  const int rows = p.B * p.S;
  if (rows == 0) return cudaSuccess;
  a.sink_k = p.sink_k; a.sink_v = p.sink_v; a.nsink = p.sink_k ? p.nsink : 0;
  a.skip_first_copy = g_arm_skip_copy.exchange(0);
  const int nkeys = a.nsink + (p.idx ? p.K : p.window);
  split_policy(rows, nkeys, &a.nsplit, &a.keys_per_split, p.idx != nullptr);
  a.key_list_bytes = ((uint32_t)a.keys_per_split * 4u + 127u) & ~127u;
  if (a.nsplit > 1) {
    const size_t need = (size_t)rows * a.nsplit * p.H * (p.DV + 2) * sizeof(float);
    if (ws == nullptr || ws_bytes < need) return cudaErrorInvalidValue;
    a.part_o = static_cast<float*>(ws);
    a.part_ml = a.part_o + (size_t)rows * a.nsplit * p.H * p.DV;
  }
  const size_t es = p.dtype == 0 ? 4 : 2;
  a.k_bytes = (uint32_t)(p.HKV * p.DQK * es);
  a.v_bytes = (uint32_t)(p.HKV * p.DV * es);
  a.slot_bytes = (a.k_bytes + a.v_bytes + 127) & ~127u;
  // as many row slots as fit while two CTAs stay resident per SM (227 KB shared memory):
  // the ring is what keeps HBM busy, a row pair being ~20 KB at the large shapes
  const size_t per_cta = (227 * 1024) / 2 - 1024 - a.key_list_bytes - 512;
  int ns = (int)(per_cta / a.slot_bytes);
  ns = ns < 2 ? 2 : (ns > 16 ? 16 : ns);
  a.nslots = ns;
  const size_t smem = 1024 + a.key_list_bytes + (size_t)ns * a.slot_bytes;
  if (smem > 227 * 1024) return cudaErrorNotSupported;
  const int hpw = heads_per_warp(p.H);
  if (hpw == 0) return cudaErrorNotSupported;
  const unsigned grid = (unsigned)(rows * a.nsplit);
  if (p.dtype == 0) return launch_hpw<float>(a, hpw, smem, grid, rows, st);
  return launch_hpw<__nv_bfloat16>(a, hpw, smem, grid, rows, st);
}

}  // namespace dsa
