// Sparse attention as dense tensor-core tiles under the selection mask (tcgen05 + TMEM +
// TMA), with the headwise gate fused; the same core computes the sliding-window layers.
//
// [AXK2] "注意力前向的骨架：MLA + 显式稀疏掩码": the indexer's top-k positions become an additive
// sparse mask folded with the causal mask into attention_mask, and attention runs densely
// under that mask (eager/SDPA) -- every unselected position contributes exp(-inf) = 0.  This
// kernel is that computation on Blackwell tensor cores: for each (batch, head, block of 128
// queries) it walks the causal key blocks of 128, computes S = Q K^T into tensor memory,
// applies the per-query selection bits (one bit per key, written by the top-k kernel), runs
// an online softmax in float32 and accumulates O += P V on the tensor cores.  [SPARK]
// "前向流程": out *= act(gate[b,s,h]) in float32 before the cast.  [PANGU] §3.2: the SWA
// layers use the same core with the band s+q_off-W < t <= s+q_off and grouped KV heads.
//
// Layout of one work item: Q block [128 x Dqk], K block [128 x Dqk] (both K-major bf16,
// 128-byte swizzle, via 3-D tensor maps over (dim, head, token)), V block [128 x Dv]
// (MN-major operand of the second product).  Tensor memory: S0, S1 (128 columns each,
// double-buffered so S_{j+1} = Q K_{j+1}^T overlaps the softmax of block j), O (Dv columns);
// P is split into bf16 P_hi + P_lo (two per 32-bit column, 64 columns each) that overwrite
// their S buffer and feed O += P_hi V + P_lo V as tensor-memory A operands -- the low part
// keeps the float32 probabilities' precision that a single bf16 P would lose.  The running max is only raised (and O, l
// rescaled) when a row's block max exceeds it by more than 2^8, so exp2 arguments stay
// <= 8 and rescales are rare.
//
// Roles: warp 0 TMA producer, warp 1 MMA issuer (one thread), warps 4..7 softmax and
// epilogue (thread = query row = TMEM lane).  Persistent CTAs take items round-robin,
// longest first.  Every wait is bounded.
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace dsa {

namespace {

constexpr int kBlk = 128;     // queries per item = keys per block
constexpr int kSoftWarp0 = 4; // softmax warps 4..7
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleLog2 = 8.0f;

struct AttnArgs {
  const uint32_t* mask;  // selection bits [B*S, mask_stride] or NULL (band mode)
  const void* gate;      // [B,S,H] bf16 or NULL
  __nv_bfloat16* out;    // [B,S,H,Dv]
  int gate_mode;
  float qk_scale;        // sm_scale * log2(e)
  int B, S, T, H, HKV, q_off, window;
  int mask_stride;       // words per mask row (multiple of 4)
  int nqb;
};

template <int DQK_, int DV_, bool BAND_>
struct FaCfg {
  static constexpr int DQK = DQK_, DV = DV_;
  static constexpr bool BAND = BAND_;
  static constexpr int QKH = DQK / 64, VH = DV / 64;
  static constexpr int SLICE = kBlk * 128;          // one 64-element slice of a 128-row tile
  static constexpr int Q_BYTES = QKH * SLICE;
  static constexpr int K_BYTES = QKH * SLICE;
  static constexpr int V_BYTES = VH * SLICE;
  static constexpr int KV_BYTES = K_BYTES + V_BYTES;
  static constexpr int STAGES = 2;
  static constexpr int SMEM = Q_BYTES + STAGES * KV_BYTES + 256 + 1024;
  static constexpr int THREADS = 32 * (kSoftWarp0 + 4);
  static constexpr int S_COLS = kBlk;              // fp32 columns of one S buffer
  static constexpr int O_COL = 2 * S_COLS;         // O starts after S0, S1
  static constexpr int TMEM_COLS = 512;
  static_assert(DQK % 64 == 0 && DV % 64 == 0 && DV <= 256, "head dims");
  static_assert(O_COL + DV <= TMEM_COLS, "TMEM budget");
};

// Instruction descriptor, kind::f16, bf16 A/B, f32 D, with the B operand MN-major.
__host__ __device__ constexpr uint32_t idesc_bf16_f32_bmn(int M, int N) {
  return idesc_bf16_f32(M, N) | (1u << 16);
}

// Shared-memory descriptor of an MN-major tile with the 128-byte swizzle: 64 MN elements
// (128 B) per swizzle row, K rows 128 B apart, 8-row atoms `sbo` apart, 64-element MN
// groups `lbo` apart.
__device__ __forceinline__ uint64_t sw128_mnmajor_desc(uint32_t start, uint32_t lbo,
                                                       uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((start & 0x3FFFF) >> 4);
  d |= (uint64_t)((lbo >> 4) & 0x3FFF) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFF) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

// 2^x on the special-function unit (flush-to-zero; exp2(-inf) = +0).
__device__ __forceinline__ float ex2_ftz(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int x, int y,
                                            int z, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
      "l"(map), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void drain(uint64_t* bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity))
    if (clock64() - t0 > kWaitCycles) {
      flag_status(kStatusTimeout);
      return;
    }
}

// Item i -> (query block, batch row, head); longest query blocks first.
struct Item {
  int qb, b, h;
};
__device__ __forceinline__ Item item_of(const AttnArgs& a, int i) {
  Item it;
  it.h = i % a.H;
  const int r = i / a.H;
  it.b = r % a.B;
  it.qb = a.nqb - 1 - r / a.B;
  return it;
}
// Key blocks [j0, j1) item `it` must visit.
template <bool BAND>
__device__ __forceinline__ void key_range(const AttnArgs& a, const Item& it, int* j0, int* j1) {
  const int s0 = it.qb * kBlk;
  const int s_last = min(a.S - 1, s0 + kBlk - 1);
  const int t_hi = min(a.T - 1, s_last + a.q_off);
  *j1 = t_hi / kBlk + 1;
  *j0 = 0;
  if (BAND) {
    const int t_lo = max(0, s0 + a.q_off - a.window + 1);
    *j0 = t_lo / kBlk;
  }
}

template <class C>
__global__ void __launch_bounds__(C::THREADS, 1)
    masked_attn_tc_kernel(const __grid_constant__ CUtensorMap qmap,
                          const __grid_constant__ CUtensorMap kmap,
                          const __grid_constant__ CUtensorMap vmap, const AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* Qs = smem;
  uint8_t* KVs = smem + C::Q_BYTES;  // [STAGES] x (K block, V block)
  uint64_t* bars = reinterpret_cast<uint64_t*>(KVs + C::STAGES * C::KV_BYTES);
  uint64_t* q_full = bars;           // 1
  uint64_t* q_empty = bars + 1;      // 1
  uint64_t* kv_full = bars + 2;      // [2]
  uint64_t* kv_empty = bars + 4;     // [2]
  uint64_t* s_full = bars + 6;       // [2]
  uint64_t* s_empty = bars + 8;      // [2]
  uint64_t* p_full = bars + 10;      // [2]
  uint64_t* pv_done = bars + 12;     // 1 (one phase per block)
  uint64_t* o_empty = bars + 13;     // 1 (one phase per item)
  uint64_t* mma_done = bars + 14;    // 1
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 15);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_items = a.B * a.H * a.nqb;
  const int group = a.H / a.HKV;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1); mbar_init(q_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&kv_full[i], 1); mbar_init(&kv_empty[i], 1);
      mbar_init(&s_full[i], 1); mbar_init(&s_empty[i], 1);
      mbar_init(&p_full[i], 4);
    }
    mbar_init(pv_done, 1); mbar_init(o_empty, 4); mbar_init(mma_done, 1);
    fence_mbar_init();
    prefetch_tmap(&qmap); prefetch_tmap(&kmap); prefetch_tmap(&vmap);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t g = 0, ni = 0;
      bool ok = true;
      for (int i = blockIdx.x; ok && i < n_items; i += gridDim.x, ++ni) {
        const Item it = item_of(a, i);
        int j0, j1;
        key_range<C::BAND>(a, it, &j0, &j1);
        if (ni > 0 && !mbar_wait(q_empty, (ni - 1) & 1)) { ok = false; break; }
        mbar_arrive_expect_tx(q_full, C::Q_BYTES);
        const int qrow = it.b * a.S + it.qb * kBlk;
#pragma unroll
        for (int x = 0; x < C::QKH; ++x)
          tma_load_3d(Qs + x * C::SLICE, &qmap, x * 64, it.h, qrow, q_full);
        const int kvh = it.h / group;
        for (int j = j0; j < j1; ++j, ++g) {
          const int st = g & 1;
          if (g >= 2 && !mbar_wait(&kv_empty[st], ((g >> 1) - 1) & 1)) { ok = false; break; }
          mbar_arrive_expect_tx(&kv_full[st], C::KV_BYTES);
          uint8_t* kdst = KVs + st * C::KV_BYTES;
          const int krow = it.b * a.T + j * kBlk;
#pragma unroll
          for (int x = 0; x < C::QKH; ++x)
            tma_load_3d(kdst + x * C::SLICE, &kmap, x * 64, kvh, krow, &kv_full[st]);
#pragma unroll
          for (int x = 0; x < C::VH; ++x)
            tma_load_3d(kdst + C::K_BYTES + x * C::SLICE, &vmap, x * 64, kvh, krow,
                        &kv_full[st]);
        }
      }
      // let the copies in flight land before exit
      if (g >= 1) drain(&kv_full[(g - 1) & 1], ((g - 1) >> 1) & 1);
      if (g >= 2) drain(&kv_full[(g - 2) & 1], ((g - 2) >> 1) & 1);
      if (ni >= 1) drain(q_full, (ni - 1) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(kBlk, kBlk);
      constexpr uint32_t idesc_pv = idesc_bf16_f32_bmn(kBlk, C::DV);
      const uint32_t q_base = smem_u32(Qs);
      uint32_t g = 0, ni = 0;
      bool ok = true;
      // S_g = Q K_g^T into S[g & 1]
      auto issue_qk = [&](uint32_t gg) -> bool {
        const int st = gg & 1;
        if (!mbar_wait(&kv_full[st], (gg >> 1) & 1)) return false;
        if (gg >= 2 && !mbar_wait(&s_empty[gg & 1], ((gg >> 1) - 1) & 1)) return false;
        tc_fence_after();
        const uint32_t k_base = smem_u32(KVs + st * C::KV_BYTES);
#pragma unroll
        for (int kk = 0; kk < C::DQK / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::SLICE + (kk & 3) * 32;
          umma_f16_ss(tmem + (gg & 1) * C::S_COLS, sw128_kmajor_desc(q_base + off),
                      sw128_kmajor_desc(k_base + off), idesc_qk, kk > 0 ? 1u : 0u);
        }
        umma_commit(&s_full[gg & 1]);
        return true;
      };
      for (int i = blockIdx.x; ok && i < n_items; i += gridDim.x, ++ni) {
        const Item it = item_of(a, i);
        int j0, j1;
        key_range<C::BAND>(a, it, &j0, &j1);
        const int nb = j1 - j0;
        if (!mbar_wait(q_full, ni & 1)) { ok = false; break; }
        if (!issue_qk(g)) { ok = false; break; }
        for (int j = 0; j < nb; ++j) {
          const uint32_t gg = g + j;
          if (j + 1 < nb && !issue_qk(gg + 1)) { ok = false; break; }
          if (j + 1 == nb) umma_commit(q_empty);  // Q free once the last S is computed
          if (!mbar_wait(&p_full[gg & 1], (gg >> 1) & 1)) { ok = false; break; }
          if (j == 0 && ni > 0 && !mbar_wait(o_empty, (ni - 1) & 1)) { ok = false; break; }
          tc_fence_after();
          const uint32_t v_base = smem_u32(KVs + (gg & 1) * C::KV_BYTES + C::K_BYTES);
          const uint32_t p_tmem = tmem + (gg & 1) * C::S_COLS;
#pragma unroll
          for (int kk = 0; kk < kBlk / 16; ++kk) {
            // 16 keys: 8 packed P columns; 16 V rows = 2 swizzle atoms of 8 rows
            const uint64_t vdesc = sw128_mnmajor_desc(v_base + kk * 2048, C::SLICE, 1024);
            umma_f16_ts(tmem + C::O_COL, p_tmem + kk * 8, vdesc, idesc_pv,
                        (j > 0 || kk > 0) ? 1u : 0u);
            umma_f16_ts(tmem + C::O_COL, p_tmem + 64 + kk * 8, vdesc, idesc_pv, 1u);
          }
          umma_commit(&kv_empty[gg & 1]);
          umma_commit(&s_empty[gg & 1]);
          umma_commit(pv_done);
        }
        g += nb;
      }
      umma_commit(mma_done);
      drain(mma_done, 0);
    }
  } else if (warp >= kSoftWarp0) {
    // ------------------------------------------------------------------ softmax + epilogue
    const int quad = warp & 3;
    const uint32_t t_lane = tmem + ((uint32_t)(quad * 32) << 16);
    const float ninf = __int_as_float(0xff800000);
    uint32_t g = 0, ni = 0;
    bool ok = true;
    for (int i = blockIdx.x; ok && i < n_items; i += gridDim.x, ++ni) {
      const Item it = item_of(a, i);
      int j0, j1;
      key_range<C::BAND>(a, it, &j0, &j1);
      const int nb = j1 - j0;
      const int s = it.qb * kBlk + quad * 32 + lane;
      const int spos = s + a.q_off;
      const bool row_ok = s < a.S;
      const uint32_t* mrow =
          (!C::BAND && row_ok) ? a.mask + ((size_t)it.b * a.S + s) * a.mask_stride : nullptr;
      float m_used = ninf, l = 0.f;
      for (int j = 0; j < nb; ++j) {
        const uint32_t gg = g + j;
        const int t0 = (j0 + j) * kBlk;
        if (!warp_wait(&s_full[gg & 1], (gg >> 1) & 1)) { ok = false; break; }
        tc_fence_after();
        uint32_t bits[4] = {0u, 0u, 0u, 0u};
        if (!C::BAND) {
          if (mrow) {
            const uint4 w4 = __ldg(reinterpret_cast<const uint4*>(mrow + (t0 >> 5)));
            bits[0] = w4.x; bits[1] = w4.y; bits[2] = w4.z; bits[3] = w4.w;
          }
        } else if (row_ok) {
          // band: spos - window < t <= spos, t < T
          const int lo = max(spos - a.window + 1, 0) - t0, hi = min(spos, a.T - 1) - t0;
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            const int a0 = max(lo - 32 * w, 0), a1 = min(hi - 32 * w, 31);
            bits[w] = a1 < a0 ? 0u
                              : ((a1 - a0 == 31) ? 0xffffffffu
                                                 : (((1u << (a1 - a0 + 1)) - 1u) << a0));
          }
        }
        // raw S row: all four TMEM reads in flight, one wait
        uint32_t r[kBlk];
        tmem_ld32(t_lane + (gg & 1) * C::S_COLS + 0, *reinterpret_cast<uint32_t(*)[32]>(r + 0));
        tmem_ld32(t_lane + (gg & 1) * C::S_COLS + 32, *reinterpret_cast<uint32_t(*)[32]>(r + 32));
        tmem_ld32(t_lane + (gg & 1) * C::S_COLS + 64, *reinterpret_cast<uint32_t(*)[32]>(r + 64));
        tmem_ld32(t_lane + (gg & 1) * C::S_COLS + 96, *reinterpret_cast<uint32_t(*)[32]>(r + 96));
        tmem_wait_ld();
        // masked raw scores (unselected -> -inf) and their max; the scale is positive, so
        // max(scale * s) = scale * max(s) and the scale folds into the exp argument below
        float x[kBlk];
        float mraw = ninf;
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            x[c * 32 + e] = (bits[c] & (1u << e)) ? __uint_as_float(r[c * 32 + e]) : ninf;
            mraw = fmaxf(mraw, x[c * 32 + e]);
          }
        const float mb = mraw * a.qk_scale;
        const bool need = mb > m_used + kRescaleLog2;
        if (__any_sync(0xffffffffu, need)) {
          const float m_new = need ? mb : m_used;
          const float alpha = (l > 0.f) ? exp2f(m_used - m_new) : 0.f;
          // O holds the previous blocks of this item: rescale it once the last P V landed
          if (j > 0 && __any_sync(0xffffffffu, need && l > 0.f)) {
            if (!warp_wait(pv_done, (gg - 1) & 1)) { ok = false; break; }
            tc_fence_after();
#pragma unroll 1
            for (int c = 0; c < C::DV / 16; ++c) {
              uint32_t r[16];
              tmem_ld16(t_lane + C::O_COL + c * 16, r);
              tmem_wait_ld();
              if (need) {
#pragma unroll
                for (int e = 0; e < 16; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
              }
              tmem_st16(t_lane + C::O_COL + c * 16, r);
            }
            tmem_wait_st();
          }
          if (need) {
            l *= alpha;
            m_used = m_new;
          }
        }
        // P = P_hi + P_lo, both bf16 (P_hi = bf16(p), P_lo = bf16(p - P_hi)): the second
        // product recovers the bits bf16 drops, so O carries ~2^-17 relative error in P
        // instead of 2^-9.  P_hi fills columns [0,64) of the S buffer, P_lo [64,128).
        float rs = 0.f;
        // exp2(scale * s - m); -inf (unselected) gives exactly 0.  With no selected key yet
        // (m_used = -inf) every x is -inf as well; subtracting 0 keeps the result 0.
        const float msub = m_used == ninf ? 0.f : m_used;
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          uint32_t ph[32], pl[32];
#pragma unroll
          for (int e2 = 0; e2 < 32; ++e2) {
            const int e = hf * 64 + 2 * e2;
            const float p0 = ex2_ftz(fmaf(x[e], a.qk_scale, -msub));
            const float p1 = ex2_ftz(fmaf(x[e + 1], a.qk_scale, -msub));
            rs += p0 + p1;
            const __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
            const float2 hf2 = __bfloat1622float2(h2);
            const __nv_bfloat162 l2 = __floats2bfloat162_rn(p0 - hf2.x, p1 - hf2.y);
            ph[e2] = *reinterpret_cast<const uint32_t*>(&h2);
            pl[e2] = *reinterpret_cast<const uint32_t*>(&l2);
          }
          tmem_st32(t_lane + (gg & 1) * C::S_COLS + hf * 32, ph);
          tmem_st32(t_lane + (gg & 1) * C::S_COLS + 64 + hf * 32, pl);
        }
        l += rs;
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[gg & 1]);
      }
      if (!ok) break;
      g += nb;
      // epilogue: O / l, gate, bf16 store
      if (!warp_wait(pv_done, (g - 1) & 1)) { ok = false; break; }
      tc_fence_after();
      float f = l > 0.f ? 1.0f / l : 0.f;
      if (a.gate && row_ok)
        f *= gate_act(__bfloat162float(
                          static_cast<const __nv_bfloat16*>(a.gate)[((size_t)it.b * a.S + s) * a.H +
                                                                   it.h]),
                      a.gate_mode);
      __nv_bfloat16* orow = a.out + (((size_t)it.b * a.S + s) * a.H + it.h) * C::DV;
#pragma unroll 1
      for (int c = 0; c < C::DV / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(t_lane + C::O_COL + c * 32, r);
        tmem_wait_ld();
        if (c == C::DV / 32 - 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(o_empty);
        }
        if (row_ok) {
          uint4 v4[4];
          uint32_t* vw = reinterpret_cast<uint32_t*>(v4);
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            __nv_bfloat162 h2 = __floats2bfloat162_rn(__uint_as_float(r[2 * e]) * f,
                                                      __uint_as_float(r[2 * e + 1]) * f);
            vw[e] = *reinterpret_cast<uint32_t*>(&h2);
          }
          uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
          for (int e = 0; e < 4; ++e) dst[e] = v4[e];
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 3-D bf16 map over [tokens, heads, dim] (dim fastest): box = 64 dims x 1 head x 128 tokens,
// 128-byte swizzle.
bool map3d(CUtensorMap* m, const void* base, uint64_t tokens, uint64_t heads, uint64_t dim) {
  auto enc = encoder();
  if (!enc) return false;
  cuuint64_t dims[3] = {dim, heads, tokens};
  cuuint64_t strides[2] = {dim * 2, heads * dim * 2};
  cuuint32_t box[3] = {64, 1, (cuuint32_t)kBlk};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

int num_sms() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

template <class C>
cudaError_t launch_fa(const AttnProblem& p, const uint32_t* mask, int mask_stride,
                      cudaStream_t st) {
  CUtensorMap qm, km, vm;
  if (!map3d(&qm, p.q, (uint64_t)p.B * p.S, p.H, C::DQK) ||
      !map3d(&km, p.k, (uint64_t)p.B * p.T, p.HKV, C::DQK) ||
      !map3d(&vm, p.v, (uint64_t)p.B * p.T, p.HKV, C::DV))
    return cudaErrorInvalidValue;
  AttnArgs a{};
  a.mask = mask; a.gate = p.gate; a.out = static_cast<__nv_bfloat16*>(p.out);
  a.gate_mode = p.gate_mode; a.qk_scale = p.sm_scale * kLog2e;
  a.B = p.B; a.S = p.S; a.T = p.T; a.H = p.H; a.HKV = p.HKV; a.q_off = p.q_off;
  a.window = p.window; a.mask_stride = mask_stride;
  a.nqb = (p.S + kBlk - 1) / kBlk;
  const int items = p.B * p.H * a.nqb;
  const int nsm = num_sms();
  const int grid = items < nsm ? items : nsm;
  auto kern = masked_attn_tc_kernel<C>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  kern<<<grid, C::THREADS, C::SMEM, st>>>(qm, km, vm, a);
  return cudaGetLastError();
}

}  // namespace

bool masked_attn_supported(int dtype, int DQK, int DV) {
  return dtype == 1 && (DQK == 128 || DQK == 192) && DV == 128;
}

cudaError_t launch_masked_attn(const AttnProblem& p, const uint32_t* mask, int mask_stride,
                               cudaStream_t st) {
  if (!masked_attn_supported(p.dtype, p.DQK, p.DV)) return cudaErrorNotSupported;
  const bool band = p.idx == nullptr && mask == nullptr;
  if (!band && mask == nullptr) return cudaErrorInvalidValue;
  if (p.DQK == 128)
    return band ? launch_fa<FaCfg<128, 128, true>>(p, mask, mask_stride, st)
                : launch_fa<FaCfg<128, 128, false>>(p, mask, mask_stride, st);
  return band ? launch_fa<FaCfg<192, 128, true>>(p, mask, mask_stride, st)
              : launch_fa<FaCfg<192, 128, false>>(p, mask, mask_stride, st);
}

}  // namespace dsa
