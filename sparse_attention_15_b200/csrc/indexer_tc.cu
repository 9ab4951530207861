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
//   warps 2, 3   idle (they complete the first warpgroup)
//   warps 4..    epilogue (a multiple of 4 warps, so that each TMEM lane quadrant -- warp % 4 --
//                has the same number of warps): tcgen05.ld of the accumulator, weighted
//                head sum, store.  In the per-head form each epilogue warp keeps the head
//                weights of its columns in registers for a whole work unit: read per tile,
//                those broadcast loads filled the load/store unit's data path (one wavefront
//                per weight, warp and tile) and held the tensor pipe back.  setmaxnreg moves
//                registers from the first warpgroup to the epilogue to make room.
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
// First epilogue warp (warp % 4 = its TMEM lane quadrant): 4 when the kernel splits its
// registers (the producer and the MMA issuer then fill a warpgroup of their own), else 2.
template <bool SPLIT>
constexpr int epi_warp0() { return SPLIT ? 4 : 2; }
constexpr int kRegsCtl = 40;  // registers of the first warpgroup after the split

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
  // the register split and the per-unit weights apply to the wide per-head prefill form
  static constexpr bool SPLIT = !CL_ && NE_ == 16;
  // threads of the plain kernel (split registers) and of the filter kernel (no split)
  static constexpr int THREADS = 32 * (epi_warp0<SPLIT>() + NE);
  static constexpr int THREADS_FILTER = 32 * (epi_warp0<false>() + NE);
  // Registers: at launch the per-thread count the SM sub-partition with the most warps
  // allows (ptxas launches a kernel that uses setmaxnreg with this maximum); the epilogue
  // warpgroups then take what the first warpgroup gives up.
  static constexpr int WARPS_PER_SMSP = (epi_warp0<SPLIT>() + NE + 3) / 4;
  static constexpr int REGS_LAUNCH_RAW = 16384 / (32 * WARPS_PER_SMSP);
  static constexpr int REGS_LAUNCH = (REGS_LAUNCH_RAW > 255 ? 255 : REGS_LAUNCH_RAW) & ~7;
  static constexpr int REGS_EPI_RAW = (REGS_LAUNCH * THREADS - 128 * kRegsCtl) / (32 * NE);
  static constexpr int REGS_EPI = (REGS_EPI_RAW > 248 ? 248 : REGS_EPI_RAW) & ~7;
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

// This CTA's work units.  Unit u = c * (B * nqb) + (b * nqb + qb) covers key tiles
// [c*chunk, min(ntiles(qb), (c+1)*chunk)); units with c >= chunks(qb) are empty and
// skipped.  CTA i takes u = i, i + G, i + 2G, ... (decoded directly, no scan).  The order is
// chunk-major: the non-empty units of a layer c are a contiguous run of query blocks, which
// the stride G spreads evenly over the CTAs, and the CTAs working together read the same
// key tiles.  (With the chunk index fastest, G = 148 -- a multiple of 4, as max_chunks
// often is -- gave CTA i only the chunks c = i mod 4, ..., and the CTAs holding the late
// chunks, which only the long query blocks have, ran out of work early.)
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
    const long long nbq = (long long)a.B * a.nqb;
    const long long total = nbq * a.max_chunks;
    for (; u < total; u += ncta) {
      const int c = (int)(u / nbq);
      const long long bq = u - (long long)c * nbq;
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
__global__ void __launch_bounds__(FILTER ? C::THREADS_FILTER : C::THREADS, 1)
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

  constexpr bool kSplit = C::SPLIT && !FILTER;
  constexpr int kEpiWarp0 = epi_warp0<kSplit>();
  // The roles.  With the register split the producer and the MMA issuer run inside the
  // first warpgroup's branch, after its setmaxnreg (ptxas gives a warpgroup its own budget
  // only for code under that instruction); without it the flat dispatch lets ptxas
  // allocate the filter form without spills.
  if constexpr (kSplit) {
    if (warp < kEpiWarp0) {
      asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsCtl));
      if (warp == 0) {
#include "indexer_tc_producer.cuh"
      } else if (warp == 1) {
#include "indexer_tc_mma.cuh"
      }
    } else {
      asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(C::REGS_EPI));
#include "indexer_tc_epilogue.cuh"
    }
  } else {
    if (warp == 0) {
#include "indexer_tc_producer.cuh"
    } else if (warp == 1) {
#include "indexer_tc_mma.cuh"
    } else if (warp >= kEpiWarp0) {
#include "indexer_tc_epilogue.cuh"
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
  if (C::SPLIT && !filter) {
    // the register split only completes if the launch holds the registers it hands out
    cudaFuncAttributes fa{};
    e = cudaFuncGetAttributes(&fa, kern);
    if (e != cudaSuccess) return e;
    if (fa.numRegs * C::THREADS < 128 * kRegsCtl + 32 * C::NE * C::REGS_EPI)
      return cudaErrorInvalidConfiguration;
  }
  kern<<<grid, filter ? C::THREADS_FILTER : C::THREADS, C::SMEM, st>>>(kmap, qmap, a);
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
