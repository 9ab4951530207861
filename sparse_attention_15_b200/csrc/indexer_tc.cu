// Lightning-indexer scores on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// [AXK2] "SK Telecom 三大改进 / 1. Sparse Gated Attention（SGA）":
//   index_score[b,s,t] = sum_h weight[b,s,h] * softmax_scale * (q[b,s,h,:] . k[b,t,:]),
// causal mask imposed while scoring.  [PANGU] §3.5 Table 1: the S^2 * N_head^I * D^I term
// that dominates prefill.
//
// The per-head dot products are one dense contraction: keys x (query, head) pairs over the
// indexer dimension.  One MMA tile is
//   D[128 keys, N = NQ*HI columns] = k_idx[t0:t0+128, :] . q_idx[(s0..s0+NQ) x heads, :]^T
// (A = the key tile, B = the query block, both K-major bf16 in shared memory with the
// 128-byte swizzle, fetched by TMA; D = float32 in tensor memory).  Because a TMEM lane is
// a key, each epilogue thread owns one key and reduces over the heads of its row in
// registers -- sum_h w[s,h] * D[t, (s,h)] -- with no cross-lane traffic, then applies the
// scale, the optional ReLU and the causal mask and writes one float per query, coalesced
// along t.
//
// Roles (persistent CTAs, one per SM; all waits bounded):
//   warp 0       TMA producer: the query block of each work unit (double-buffered) and a
//                ring of key tiles
//   warp 1       MMA issuer (one thread): DI/16 tcgen05.mma per tile into one of two TMEM
//                accumulators; tcgen05.commit frees the key stage and hands the
//                accumulator to the epilogue
//   warps 2..    epilogue (a multiple of 4 warps, so that each TMEM lane quadrant -- warp % 4 --
//                has the same number of warps): tcgen05.ld of the accumulator, weighted
//                head sum, store
// A work unit is (batch row, query block, a chunk of key tiles up to the causal limit);
// units are dealt to CTAs round-robin.  Key tiles after the last causal tile of a query
// block are not computed: a separate fill kernel writes their -inf when asked to.
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace dsa {

namespace {

constexpr int kTileM = 128;   // keys per tile = TMEM lanes
constexpr int kEpiWarp0 = 2;  // first epilogue warp (warp % 4 = its TMEM lane quadrant)

struct TcArgs {
  const float* w;
  float* scores;
  float scale;
  int B, S, T, q_off;
  int nqb;         // query blocks per batch row
  int chunk;       // key tiles per work unit
  int max_chunks;  // units per query block slot (chunks of the longest block)
  // Key tile kt of a unit is key tile kt * kstride of the row (1: every tile; > 1: a strided
  // sample of the tiles).  Scores land in column kt * 128 + r of rows ldT floats long.
  int kstride;
  long long ldT;
  // Filter mode (tau != NULL): instead of storing scores, append every causal key whose
  // order key is >= tau[row] to the row's candidate list (order key, key index) -- the first
  // cand_cap of them; cand_cnt[row] counts all of them.
  const uint32_t* tau;
  uint2* cand;
  int* cand_cnt;
  int cand_cap;
  // If non-NULL, the launch does nothing unless *run_if != 0 (set on the device by an
  // earlier kernel of the stream).
  const int* run_if;
};

// CL_: the head-collapsed form -- the B operand holds two bf16 rows per query (the hi and
// lo parts of sum_h w[s,h] q_I[s,h,:]) and a score is the sum of its two columns.
// ES_: operand element bytes, 2 (bf16, kind::f16) or 1 (e4m3, kind::f8f6f4).  Every MMA
// consumes 32 bytes of each 128-byte swizzled row either way, so the shared-memory layout
// and the descriptor arithmetic are the same in bytes.
// NACC_: TMEM accumulators (2 or 4): with more, the MMA runs further ahead of the epilogue.
template <int HI_, int DI_, int NQ_, int NE_, int NA_, int NB_ = 2, bool CL_ = false,
          int ES_ = 2, int NACC_ = 2>
struct TcCfg {
  static constexpr int HI = HI_, DI = DI_, NQ = NQ_, NE = NE_, NA = NA_;
  static constexpr bool CL = CL_;
  static constexpr int ES = ES_;
  static constexpr int ROW_BYTES = DI * ES;       // one operand row
  static constexpr int SLICE_ELEMS = 128 / ES;    // elements per 128-byte swizzle row
  static constexpr int NB = NB_;                  // query-block buffers (1 or 2)
  static constexpr int N = NQ * HI;               // MMA N: (query, head) columns
  static constexpr int KH = ROW_BYTES / 128;      // 128-byte K slices
  static constexpr int A_SLICE = kTileM * 128;    // bytes of one K slice of a key tile
  static constexpr int A_BYTES = KH * A_SLICE;
  static constexpr int B_SLICE = N * 128;
  static constexpr int B_BYTES = KH * B_SLICE;
  static constexpr int NACC = NACC_;
  static constexpr int ACC_COLS = N;              // one accumulator
  static constexpr int TMEM_COLS = NACC * N <= 32 ? 32 : NACC * N <= 64 ? 64
                                   : NACC * N <= 128 ? 128 : NACC * N <= 256 ? 256 : 512;
  static constexpr int EPI_GROUPS = NE / 4;       // epilogue warps per TMEM lane quadrant
  static constexpr int COLS_PER_WARP = N / EPI_GROUPS;
  static constexpr int THREADS = 32 * (kEpiWarp0 + NE);
  static constexpr int BAR_BYTES = 256;
  static constexpr int SMEM = NA * A_BYTES + NB * B_BYTES + BAR_BYTES + 1024;
  static_assert(N % 16 == 0 && N >= 16 && N <= 256, "UMMA N");
  static_assert((NACC == 2 || NACC == 4) && NACC * N <= 512, "accumulators must fit TMEM");
  static_assert(HI <= 32 && 32 % HI == 0, "heads per 32-column chunk");
  static_assert(!CL || HI == 2, "the collapsed form has two columns (hi, lo) per query");
  static_assert(CL || HI >= 16, "per-head epilogue: a query spans whole 16-column chunks");
  static_assert(COLS_PER_WARP % 32 == 0 && COLS_PER_WARP % HI == 0, "epilogue chunking");
  static_assert(ROW_BYTES % 128 == 0, "operand rows must be whole 128-byte slices");
  static_assert(ES == 2 || (ES == 1 && !CL), "e4m3 operands: per-head form only");
};

// This CTA's work units.  Unit u = (b * nqb + qb) * max_chunks + c covers key tiles
// [c*chunk, min(ntiles(qb), (c+1)*chunk)); units with c >= chunks(qb) are empty and
// skipped.  CTA i takes u = i, i + G, i + 2G, ... (decoded directly, no scan).
struct UnitIter {
  long long u;
  int b = 0, qb = 0, k0 = 0, k1 = 0;
  __device__ __forceinline__ explicit UnitIter(int cta) : u((long long)cta) {}
  __device__ __forceinline__ static int ntiles(const TcArgs& a, int q, int NQ) {
    const int s_last = min(a.S - 1, q * NQ + NQ - 1);
    const int t_last = min(a.T - 1, s_last + a.q_off);
    return (t_last / kTileM) / a.kstride + 1;
  }
  // Next non-empty unit owned by this CTA; false when done.
  __device__ __forceinline__ bool next(const TcArgs& a, int NQ, int ncta) {
    const long long total = (long long)a.B * a.nqb * a.max_chunks;
    for (; u < total; u += ncta) {
      const int c = (int)(u % a.max_chunks);
      const long long bq = u / a.max_chunks;
      qb = (int)(bq % a.nqb);
      b = (int)(bq / a.nqb);
      const int nt = ntiles(a, qb, NQ);
      k0 = c * a.chunk;
      if (k0 >= nt) continue;
      k1 = min(nt, k0 + a.chunk);
      u += ncta;
      return true;
    }
    return false;
  }
};

template <class C, int RELU, bool FILTER>
__global__ void __launch_bounds__(C::THREADS, 1)
    index_scores_tc_kernel(const __grid_constant__ CUtensorMap kmap,
                           const __grid_constant__ CUtensorMap qmap, const TcArgs a) {
  // a launch kept for a fallback that was not needed: every thread leaves at once
  if (a.run_if != nullptr && *reinterpret_cast<const volatile int*>(a.run_if) == 0) return;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* As = smem;                               // NA key tiles
  uint8_t* Bs = smem + C::NA * C::A_BYTES;          // NB query blocks
  uint64_t* bars = reinterpret_cast<uint64_t*>(Bs + C::NB * C::B_BYTES);
  uint64_t* a_full = bars;                          // [NA]
  uint64_t* a_empty = a_full + C::NA;               // [NA]
  uint64_t* b_full = a_empty + C::NA;               // [2]
  uint64_t* b_empty = b_full + 2;                   // [2]
  uint64_t* acc_full = b_empty + 2;                 // [NACC]
  uint64_t* acc_empty = acc_full + C::NACC;         // [NACC]
  uint64_t* mma_done = acc_empty + C::NACC;         // [1]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cta = blockIdx.x, ncta = gridDim.x;  // persistent CTAs

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NA; ++i) { mbar_init(&a_full[i], 1); mbar_init(&a_empty[i], 1); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&b_full[i], 1); mbar_init(&b_empty[i], 1);
    }
    for (int i = 0; i < C::NACC; ++i) {
      mbar_init(&acc_full[i], 1); mbar_init(&acc_empty[i], C::NE);
    }
    mbar_init(mma_done, 1);
    fence_mbar_init();
    prefetch_tmap(&kmap);
    prefetch_tmap(&qmap);
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
      UnitIter it(cta);
      uint32_t ai = 0, bi = 0;
      bool ok = true;
      while (ok && it.next(a, C::NQ, ncta)) {
        const int bb = bi % C::NB;
        if (bi >= (uint32_t)C::NB && !mbar_wait(&b_empty[bb], ((bi / C::NB) - 1) & 1)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&b_full[bb], C::B_BYTES);
        const int qrow = (it.b * a.S + it.qb * C::NQ) * C::HI;
#pragma unroll
        for (int kh = 0; kh < C::KH; ++kh)
          tma_load_2d(Bs + bb * C::B_BYTES + kh * C::B_SLICE, &qmap, kh * C::SLICE_ELEMS, qrow,
                      &b_full[bb]);
        ++bi;
        for (int kt = it.k0; kt < it.k1; ++kt) {
          const int st = ai % C::NA;
          if (ai >= (uint32_t)C::NA && !mbar_wait(&a_empty[st], ((ai / C::NA) - 1) & 1)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&a_full[st], C::A_BYTES);
          const int krow = it.b * a.T + kt * a.kstride * kTileM;
#pragma unroll
          for (int kh = 0; kh < C::KH; ++kh)
            tma_load_2d(As + st * C::A_BYTES + kh * C::A_SLICE, &kmap, kh * C::SLICE_ELEMS, krow,
                        &a_full[st]);
          ++ai;
        }
      }
      // on the way out, let every copy this thread issued land
      for (uint32_t j = (ai > (uint32_t)C::NA ? ai - C::NA : 0); j < ai; ++j)
        drain_wait(&a_full[j % C::NA], (j / C::NA) & 1);
      for (uint32_t j = (bi > (uint32_t)C::NB ? bi - C::NB : 0); j < bi; ++j)
        drain_wait(&b_full[j % C::NB], (j / C::NB) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc =
          C::ES == 2 ? idesc_bf16_f32(kTileM, C::N) : idesc_e4m3_f32(kTileM, C::N);
      UnitIter it(cta);
      uint32_t ai = 0, bi = 0, ci = 0;
      bool ok = true;
      while (ok && it.next(a, C::NQ, ncta)) {
        const int bb = bi % C::NB;
        if (!mbar_wait(&b_full[bb], (bi / C::NB) & 1)) { ok = false; break; }
        const uint32_t b_base = smem_u32(Bs + bb * C::B_BYTES);
        for (int kt = it.k0; kt < it.k1; ++kt) {
          const int st = ai % C::NA;
          if (!mbar_wait(&a_full[st], (ai / C::NA) & 1)) { ok = false; break; }
          const int ab = ci % C::NACC;
          if (ci >= (uint32_t)C::NACC &&
              !mbar_wait(&acc_empty[ab], ((ci / C::NACC) - 1) & 1)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_base = smem_u32(As + st * C::A_BYTES);
#pragma unroll
          for (int kk = 0; kk < C::ROW_BYTES / 32; ++kk) {
            const uint32_t off = (kk & 3) * 32;  // 32 B (16 bf16 / 32 e4m3) along the row
            const uint64_t adesc = sw128_kmajor_desc(a_base + (kk >> 2) * C::A_SLICE + off);
            const uint64_t bdesc = sw128_kmajor_desc(b_base + (kk >> 2) * C::B_SLICE + off);
            if constexpr (C::ES == 2)
              umma_f16_ss(tmem + ab * C::ACC_COLS, adesc, bdesc, idesc, kk > 0 ? 1u : 0u);
            else
              umma_f8f6f4_ss(tmem + ab * C::ACC_COLS, adesc, bdesc, idesc, kk > 0 ? 1u : 0u);
          }
          umma_commit(&a_empty[st]);
          umma_commit(&acc_full[ab]);
          ++ai;
          ++ci;
        }
        if (!ok) break;
        umma_commit(&b_empty[bb]);
        ++bi;
      }
      umma_commit(mma_done);
      drain_wait(mma_done, 0);
    }
  } else if (warp >= kEpiWarp0) {
    // ------------------------------------------------------------------ epilogue
    const int ew = warp - kEpiWarp0;
    const int quad = warp & 3;
    const int group = ew >> 2;
    const int col0 = group * C::COLS_PER_WARP;
    const uint32_t t_lane = tmem + ((uint32_t)(quad * 32) << 16);
    const float ninf = __int_as_float(0xff800000);
    UnitIter it(cta);
    uint32_t ci = 0;
    bool ok = true;
    // Filter mode: the candidates of each of this warp's queries found in one key tile are
    // written when that query comes round again in the next tile (or at the end of the
    // unit): the list position comes from a global atomicAdd issued when the scores are
    // ready, and its round trip overlaps the next tile's work instead of stalling this one.
    constexpr int QW = C::CL ? 1 : (C::COLS_PER_WARP / C::HI);  // queries per warp and tile
    struct Pending {
      uint32_t bal, key;
      int t, base;
      size_t off;
    };
    Pending pend[QW];
    uint32_t tau_q[QW];
#pragma unroll
    for (int q = 0; q < QW; ++q) pend[q].bal = 0u;
    const uint32_t lt_mask = (1u << lane) - 1u;
    auto flush = [&](Pending& p) {  // p.bal is warp-uniform
      if (p.bal) {
        const int base = __shfl_sync(0xffffffffu, p.base, 0);
        const int pos = base + __popc(p.bal & lt_mask);
        if (((p.bal >> lane) & 1u) && pos < a.cand_cap)
          a.cand[p.off + pos] = make_uint2(p.key, (uint32_t)p.t);
        p.bal = 0u;
      }
    };
    while (ok && it.next(a, C::NQ, ncta)) {
      const int s_base = it.qb * C::NQ;
      if constexpr (FILTER) {
#pragma unroll
        for (int q = 0; q < QW; ++q) {
          flush(pend[q]);
          const int sq = s_base + col0 / C::HI + q;
          tau_q[q] = sq < a.S ? __ldg(a.tau + (size_t)it.b * a.S + sq) : 0xffffffffu;
        }
      }
      // the head weights of this unit's queries (1-2 KB) are the same for every key tile and
      // every lane: the reduction reads them as warp-wide broadcast float4 loads, which stay
      // in L1 for the whole unit (one load per four heads, no shuffles)
      const float4* wunit = C::CL ? nullptr : reinterpret_cast<const float4*>(
          a.w + ((size_t)it.b * a.S + s_base) * C::HI);
      for (int kt = it.k0; kt < it.k1; ++kt) {
        const int ab = ci % C::NACC;
        if (!warp_wait(&acc_full[ab], (ci / C::NACC) & 1)) { ok = false; break; }
        tc_fence_after();
        const int tcol = kt * kTileM + quad * 32 + lane;  // output column
        const int t = kt * a.kstride * kTileM + quad * 32 + lane;  // key position
        constexpr int NCH = C::COLS_PER_WARP / 16;
        // double-buffered 16-column TMEM reads: chunk cc+1 is in flight while chunk cc is
        // reduced.  A query's HI columns span HI/16 chunks; its four FMA chains carry over.
        uint32_t rb[2][16];
        tmem_ld16(t_lane + ab * C::ACC_COLS + col0, rb[0]);
        tmem_wait_ld();
        // four independent FMA chains (heads h % 4) as two packed float32 pairs
        unsigned long long acc01 = pack2(0.f, 0.f), acc23 = pack2(0.f, 0.f);
#pragma unroll
        for (int cc = 0; cc < NCH; ++cc) {
          if (cc + 1 < NCH) {
            tmem_ld16(t_lane + ab * C::ACC_COLS + col0 + (cc + 1) * 16, rb[(cc + 1) & 1]);
          } else {
            // every column of this accumulator has been read: hand it back to the MMA
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[ab]);
          }
          const uint32_t* r = rb[cc & 1];
          const int c0 = col0 + cc * 16;     // first column of the chunk
          if constexpr (C::CL) {
            // eight queries per chunk: score = scale * (D[t, hi] + D[t, lo])
            const int sq = s_base + c0 / 2;
            float* op = a.scores + ((size_t)it.b * a.S + sq) * a.ldT + tcol;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              if (sq + q < a.S && t < a.T) {
                float v = (__uint_as_float(r[2 * q]) + __uint_as_float(r[2 * q + 1])) * a.scale;
                if (RELU == 1) v = fmaxf(v, 0.f);
                op[(size_t)q * a.ldT] = (t <= sq + q + a.q_off) ? v : ninf;
              }
            }
          } else {
            const int j = c0 / C::HI;          // query within the block
            const int s = s_base + j;
            if (s < a.S) {  // ragged tail of the last block (warp-uniform)
#pragma unroll
              for (int h = 0; h < 16; h += 4) {
                const float4 w4 = __ldg(wunit + (c0 + h) / 4);
                float d0 = __uint_as_float(r[h + 0]);
                float d1 = __uint_as_float(r[h + 1]);
                float d2 = __uint_as_float(r[h + 2]);
                float d3 = __uint_as_float(r[h + 3]);
                if (RELU == 2) {
                  d0 = fmaxf(d0, 0.f); d1 = fmaxf(d1, 0.f); d2 = fmaxf(d2, 0.f);
                  d3 = fmaxf(d3, 0.f);
                }
                acc01 = fma2(pack2(w4.x, w4.y), pack2(d0, d1), acc01);
                acc23 = fma2(pack2(w4.z, w4.w), pack2(d2, d3), acc23);
              }
              if ((c0 + 16) % C::HI == 0) {  // the query's last chunk: finish and store
                float a0, a1, a2, a3;
                unpack2(acc01, a0, a1);
                unpack2(acc23, a2, a3);
                float v = ((a0 + a1) + (a2 + a3)) * a.scale;
                if (RELU == 1) v = fmaxf(v, 0.f);
                const size_t row = (size_t)it.b * a.S + s;
                if constexpr (FILTER) {
                  // candidates of this query among the warp's 32 keys: one atomic per warp,
                  // the writes deferred to this query's next tile
                  Pending& p = pend[(cc * 16) / C::HI];  // compile-time slot
                  flush(p);
                  const uint32_t key = order_key(v);
                  const bool keep =
                      t < a.T && t <= s + a.q_off && key >= tau_q[(cc * 16) / C::HI];
                  p.bal = __ballot_sync(0xffffffffu, keep);
                  p.key = key;
                  p.t = t;
                  p.off = row * (size_t)a.cand_cap;
                  p.base = 0;
                  if (p.bal && lane == 0) p.base = atomicAdd(a.cand_cnt + row, __popc(p.bal));
                } else if (t < a.T) {
                  a.scores[row * a.ldT + tcol] = (t <= s + a.q_off) ? v : ninf;
                }
                acc01 = acc23 = pack2(0.f, 0.f);
              }
            }
          }
          if (cc + 1 < NCH) tmem_wait_ld();
        }
        ++ci;
      }
    }
    if constexpr (FILTER) {
#pragma unroll
      for (int q = 0; q < QW; ++q) flush(pend[q]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// -inf for the keys after the last causal tile of each query block (row-wise fill).
__global__ void fill_masked_kernel(float* __restrict__ scores, int S, int T, int q_off, int NQ) {
  const size_t row = blockIdx.x;
  const int s = (int)(row % (size_t)S);
  const int qb = s / NQ;
  const int s_last = min(S - 1, qb * NQ + NQ - 1);
  const int t_last = min(T - 1, s_last + q_off);
  const int start = (t_last / kTileM + 1) * kTileM;
  float* r = scores + row * (size_t)T;
  const float ninf = __int_as_float(0xff800000);
  for (int t = start + threadIdx.x; t < T; t += blockDim.x) r[t] = ninf;
}

// The head-collapsed query of each row: qc = sum_h w[s,h] * q_I[s,h,:] in float32 (heads in
// order), stored as two bf16 rows, hi = bf16(qc) and lo = bf16(qc - hi), so that
// k . hi + k . lo carries qc to about 2^-17 relative precision (exactly, for the integer
// workloads, where lo = 0).  One warp per row; lane l owns dims l*E .. l*E+E-1.
// E consecutive bf16 <-> float (E = 2 or 4; 4- or 8-byte aligned accesses).
template <int E>
__device__ __forceinline__ void load_bf16(const __nv_bfloat16* p, float (&x)[E]) {
  if constexpr (E == 4) {
    load4(p, x);
  } else {
    const uint32_t v = *reinterpret_cast<const uint32_t*>(p);
    x[0] = __uint_as_float(v << 16);
    x[1] = __uint_as_float(v & 0xffff0000u);
  }
}
template <int E>
__device__ __forceinline__ void store_bf16(__nv_bfloat16* p, const __nv_bfloat16 (&x)[E]) {
  uint32_t u[E / 2];
#pragma unroll
  for (int i = 0; i < E / 2; ++i)
    u[i] = (uint32_t)__bfloat16_as_ushort(x[2 * i]) |
           ((uint32_t)__bfloat16_as_ushort(x[2 * i + 1]) << 16);
  if constexpr (E == 4)
    *reinterpret_cast<uint2*>(p) = make_uint2(u[0], u[1]);
  else
    *reinterpret_cast<uint32_t*>(p) = u[0];
}

template <int DI>
__global__ void collapse_q_kernel(const __nv_bfloat16* __restrict__ q, const float* __restrict__ w,
                                  __nv_bfloat16* __restrict__ qc, long long rows, int HI) {
  constexpr int E = DI / 32;
  const long long row = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  float acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] = 0.f;
  const __nv_bfloat16* qr = q + row * HI * DI + lane * E;
  const float* wr = w + row * HI;
  for (int h = 0; h < HI; ++h) {
    const float wh = __ldg(wr + h);
    float x[E];
    load_bf16<E>(qr + (size_t)h * DI, x);
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = fmaf(wh, x[e], acc[e]);
  }
  __nv_bfloat16 hi[E], lo[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    hi[e] = __float2bfloat16_rn(acc[e]);
    lo[e] = __float2bfloat16_rn(acc[e] - __bfloat162float(hi[e]));
  }
  store_bf16<E>(qc + (row * 2) * DI + lane * E, hi);
  store_bf16<E>(qc + (row * 2 + 1) * DI + lane * E, lo);
}

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
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

// 2-D tensor map over a [rows, cols] row-major matrix of `es`-byte elements (bf16 or
// e4m3 bytes), box [128 bytes of columns, box_rows], 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows,
              int es = 2) {
  auto enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * (uint64_t)es};
  cuuint32_t box[2] = {(cuuint32_t)(128 / es), box_rows};
  cuuint32_t estr[2] = {1, 1};
  const CUtensorMapDataType dt =
      es == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8;
  CUresult r = enc(m, dt, 2, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

template <class C>
cudaError_t launch_cfg(const void* q_idx, const void* k_idx, const float* w, float scale,
                       int relu, int B, int S, int T, int q_off, float* scores,
                       int write_masked, cudaStream_t st, const IndexerExtra* ex = nullptr) {
  const IndexerExtra none{};
  const IndexerExtra& x = ex ? *ex : none;
  const int ks = x.kstride > 0 ? x.kstride : 1;
  CUtensorMap kmap, qmap;
  if (!make_map(&kmap, k_idx, (uint64_t)B * T, C::DI, kTileM, C::ES))
    return cudaErrorInvalidValue;
  if (!make_map(&qmap, q_idx, (uint64_t)B * S * C::HI, C::DI, C::N, C::ES))
    return cudaErrorInvalidValue;
  TcArgs a{};
  a.w = w; a.scores = scores; a.scale = scale; a.B = B; a.S = S; a.T = T; a.q_off = q_off;
  a.nqb = (S + C::NQ - 1) / C::NQ;
  a.kstride = ks;
  a.ldT = x.ldT > 0 ? x.ldT : T;
  a.tau = x.tau; a.cand = x.cand; a.cand_cnt = x.cand_cnt;
  a.cand_cap = x.cand_cap; a.run_if = x.run_if;
  const bool filter = x.tau != nullptr;
  // total causal tiles -> chunk size giving each CTA several units
  long long tiles = 0;
  int max_nt = 1;
  for (int qb = 0; qb < a.nqb; ++qb) {
    const int s_last = S - 1 < qb * C::NQ + C::NQ - 1 ? S - 1 : qb * C::NQ + C::NQ - 1;
    const int t_last = T - 1 < s_last + q_off ? T - 1 : s_last + q_off;
    const int nt = (t_last / kTileM) / ks + 1;
    tiles += nt;
    if (nt > max_nt) max_nt = nt;
  }
  tiles *= B;
  const int nsm = sm_count();
  long long ch = tiles / ((long long)nsm * 4);
  a.chunk = (int)(ch < 4 ? 4 : (ch > 32 ? 32 : ch));
  a.max_chunks = (max_nt + a.chunk - 1) / a.chunk;
  long long units = 0;
  for (int qb = 0; qb < a.nqb; ++qb) {
    const int s_last = S - 1 < qb * C::NQ + C::NQ - 1 ? S - 1 : qb * C::NQ + C::NQ - 1;
    const int t_last = T - 1 < s_last + q_off ? T - 1 : s_last + q_off;
    units += ((t_last / kTileM) / ks + 1 + a.chunk - 1) / a.chunk;
  }
  units *= B;
  const int grid = (int)(units < nsm ? units : nsm);
  auto kern = filter ? (relu == 1 ? index_scores_tc_kernel<C, 1, true>
                                   : (relu == 2 ? index_scores_tc_kernel<C, 2, true>
                                                : index_scores_tc_kernel<C, 0, true>))
                     : (relu == 1 ? index_scores_tc_kernel<C, 1, false>
                                  : (relu == 2 ? index_scores_tc_kernel<C, 2, false>
                                               : index_scores_tc_kernel<C, 0, false>));
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  kern<<<grid, C::THREADS, C::SMEM, st>>>(kmap, qmap, a);
  e = cudaGetLastError();
  if (e != cudaSuccess || !write_masked || filter || ks != 1) return e;
  fill_masked_kernel<<<(unsigned)((size_t)B * S), 256, 0, st>>>(scores, S, T, q_off, C::NQ);
  return cudaGetLastError();
}

}  // namespace

bool index_scores_e4m3_supported(int HI, int DI) {
  return (HI == 16 || HI == 32) && DI == 128;
}

cudaError_t launch_index_scores_e4m3(const void* q_idx, const void* k_idx, const float* w,
                                     float scale, int relu, int B, int S, int T, int HI, int DI,
                                     int q_off, float* scores, int write_masked,
                                     cudaStream_t st) {
  if (!index_scores_e4m3_supported(HI, DI)) return cudaErrorNotSupported;
  // one 128-byte slice per operand row: half the shared memory of the bf16 tiles, so the
  // key ring is deeper
  if (S == 1) {
    if (HI == 32)
      return launch_cfg<TcCfg<32, 128, 1, 4, 8, 2, false, 1>>(q_idx, k_idx, w, scale, relu, B, S,
                                                              T, q_off, scores, write_masked, st);
    return launch_cfg<TcCfg<16, 128, 2, 4, 8, 2, false, 1>>(q_idx, k_idx, w, scale, relu, B, S, T,
                                                            q_off, scores, write_masked, st);
  }
  if (HI == 32)
    return launch_cfg<TcCfg<32, 128, 8, 16, 6, 2, false, 1>>(q_idx, k_idx, w, scale, relu, B, S,
                                                             T, q_off, scores, write_masked, st);
  return launch_cfg<TcCfg<16, 128, 16, 16, 6, 2, false, 1>>(q_idx, k_idx, w, scale, relu, B, S, T,
                                                            q_off, scores, write_masked, st);
}

bool index_scores_collapsed_supported(int dtype, int DI, int relu) {
  return dtype == 1 && (DI == 64 || DI == 128) && relu != 2;
}

cudaError_t launch_collapse_q(const void* q_idx, const float* w, long long rows, int HI, int DI,
                              void* qc, cudaStream_t st) {
  if (rows <= 0) return cudaSuccess;
  const unsigned grid = (unsigned)((rows + 7) / 8);  // 8 rows (warps) per CTA
  if (DI == 128)
    collapse_q_kernel<128><<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(q_idx), w,
                                                 static_cast<__nv_bfloat16*>(qc), rows, HI);
  else if (DI == 64)
    collapse_q_kernel<64><<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(q_idx), w,
                                                static_cast<__nv_bfloat16*>(qc), rows, HI);
  else
    return cudaErrorNotSupported;
  return cudaGetLastError();
}

cudaError_t launch_index_scores_collapsed(const void* qc, const void* k_idx, float scale,
                                          int relu, int B, int S, int T, int DI, int q_off,
                                          float* scores, int write_masked, cudaStream_t st,
                                          const IndexerExtra* ex) {
  if (!index_scores_collapsed_supported(1, DI, relu)) return cudaErrorNotSupported;
  if (ex && ex->tau) return cudaErrorNotSupported;  // the filter is a per-head epilogue
  // 128 queries x (hi, lo) = 256 columns per tile
  if (DI == 128)
    return launch_cfg<TcCfg<2, 128, 128, 16, 3, 2, true>>(qc, k_idx, nullptr, scale, relu, B, S,
                                                          T, q_off, scores, write_masked, st, ex);
  return launch_cfg<TcCfg<2, 64, 128, 16, 4, 2, true>>(qc, k_idx, nullptr, scale, relu, B, S, T,
                                                       q_off, scores, write_masked, st, ex);
}

bool index_scores_tc_supported(int dtype, int HI, int DI) {
  return dtype == 1 && (HI == 16 || HI == 32) && (DI == 64 || DI == 128);
}

cudaError_t launch_index_scores_tc(const void* q_idx, const void* k_idx, const float* w,
                                   float scale, int relu, int B, int S, int T, int HI, int DI,
                                   int q_off, float* scores, int write_masked,
                                   cudaStream_t st, const IndexerExtra* ex) {
  if (!index_scores_tc_supported(1, HI, DI)) return cudaErrorNotSupported;
  if (S == 1) {  // decode: one query per batch row, N = HI, deep key pipeline
    if (HI == 32 && DI == 128)
      return launch_cfg<TcCfg<32, 128, 1, 4, 6>>(q_idx, k_idx, w, scale, relu, B, S, T, q_off,
                                                 scores, write_masked, st, ex);
    if (HI == 32 && DI == 64)
      return launch_cfg<TcCfg<32, 64, 1, 4, 8>>(q_idx, k_idx, w, scale, relu, B, S, T, q_off,
                                                scores, write_masked, st, ex);
    if (HI == 16 && DI == 128)
      return launch_cfg<TcCfg<16, 128, 2, 4, 6>>(q_idx, k_idx, w, scale, relu, B, S, T, q_off,
                                                 scores, write_masked, st, ex);
    return launch_cfg<TcCfg<16, 64, 2, 4, 8>>(q_idx, k_idx, w, scale, relu, B, S, T, q_off,
                                              scores, write_masked, st, ex);
  }
  if (HI == 32 && DI == 128)
    return launch_cfg<TcCfg<32, 128, 8, 16, 3>>(q_idx, k_idx, w, scale, relu, B, S, T, q_off,
                                               scores, write_masked, st, ex);
  if (HI == 32 && DI == 64)
    return launch_cfg<TcCfg<32, 64, 8, 16, 4>>(q_idx, k_idx, w, scale, relu, B, S, T, q_off,
                                              scores, write_masked, st, ex);
  if (HI == 16 && DI == 128)
    return launch_cfg<TcCfg<16, 128, 16, 16, 3>>(q_idx, k_idx, w, scale, relu, B, S, T, q_off,
                                                scores, write_masked, st, ex);
  // N = 128 columns (8 queries): four accumulators in TMEM keep the epilogue's latency hidden
  return launch_cfg<TcCfg<16, 64, 8, 16, 4, 2, false, 2, 4>>(q_idx, k_idx, w, scale, relu, B, S,
                                                             T, q_off, scores, write_masked, st, ex);
}

}  // namespace dsa
