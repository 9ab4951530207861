// Per-query top-k of the indexer scores.
//
// [AXK2] SGA: the indexer returns int32 indices [B, S, topk] of the keys each query keeps;
// "AXK2Config" (index_topk): topk = min(index_topk, number of keys).  [PANGU] §3.3: the
// number of selected keys is a fixed K.
//
// Order: higher score first, then lower key index (-0.0 == +0.0).  Output: the selected
// keys in ascending index order, then -1 padding.  The selection is exact: a radix select
// on order-preserving 32-bit keys (digits of 11, 11 and 10 bits, most significant first)
// finds the threshold key tau and the number `need` of keys equal to tau that still fit;
// an ordered compaction pass then keeps every key > tau and the first `need` keys == tau.
//
// One CTA per query row.  Pass 1 reads the row from HBM; the later passes re-read it from
// L2 (a row is at most a few hundred KB and was just touched).  Histograms are built with
// shared-memory atomics.  The compaction is a block-wide ballot/popc scan in index order, so
// the output is deterministic and needs no sort.  The same ballots give the selection
// bitmask (one bit per key) for the masked-tile attention path.
#include <cstring>

#include "common.cuh"
#include "kernels.h"

namespace dsa {

namespace {

constexpr int kBins = 2048;

// Block-wide exclusive prefix sum of one int per thread (blockDim.x <= 1024).
__device__ __forceinline__ int block_excl_scan(int v, int* warp_buf, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nwarps = blockDim.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_buf[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int wv = lane < nwarps ? warp_buf[lane] : 0;
    int ws = wv;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, ws, o);
      if (lane >= o) ws += y;
    }
    if (lane < nwarps) warp_buf[lane] = ws - wv;  // exclusive warp offsets
    if (lane == 31) *total = ws;
  }
  __syncthreads();
  // callers pass a barrier before the next scan rewrites warp_buf
  return warp_buf[warp] + x - v;
}

// The same scan over two ints per thread at once (one pair of barriers for both).  The block
// totals go through shared memory (*total_s): every thread reads them after the last barrier.
__device__ __forceinline__ void block_excl_scan2(int v0, int v1, int2* warp_buf2, int2* total_s,
                                                 int* ex0, int* ex1, int* total0, int* total1) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nwarps = blockDim.x >> 5;
  int x0 = v0, x1 = v1;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y0 = __shfl_up_sync(0xffffffffu, x0, o);
    const int y1 = __shfl_up_sync(0xffffffffu, x1, o);
    if (lane >= o) {
      x0 += y0;
      x1 += y1;
    }
  }
  if (lane == 31) warp_buf2[warp] = make_int2(x0, x1);
  __syncthreads();
  if (warp == 0) {
    const int2 wv = lane < nwarps ? warp_buf2[lane] : make_int2(0, 0);
    int s0 = wv.x, s1 = wv.y;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y0 = __shfl_up_sync(0xffffffffu, s0, o);
      const int y1 = __shfl_up_sync(0xffffffffu, s1, o);
      if (lane >= o) {
        s0 += y0;
        s1 += y1;
      }
    }
    if (lane < nwarps) warp_buf2[lane] = make_int2(s0 - wv.x, s1 - wv.y);
    if (lane == 31) *total_s = make_int2(s0, s1);
  }
  __syncthreads();
  const int2 off = warp_buf2[warp];
  const int2 tot = *total_s;
  *ex0 = off.x + x0 - v0;
  *ex1 = off.y + x1 - v1;
  *total0 = tot.x;
  *total1 = tot.y;
}

// Histogram bins are stored with one padding word per 32 bins, so that the contiguous runs
// of 1..16 bins each thread scans in find_bucket start in distinct banks.
constexpr int padded(int nbins) { return nbins + nbins / 32; }
__device__ __forceinline__ uint32_t hpad(uint32_t b) { return b + (b >> 5); }

template <int NT>
__device__ __forceinline__ void hist_add(uint32_t* hist, uint32_t digit, bool valid) {
  // Plain shared-memory atomics: equal digits within a warp serialise in the atomic unit,
  // which costs less than grouping them first (__match_any_sync occupies the XU pipe for
  // many cycles per call).
  if (valid) atomicAdd(&hist[hpad(digit)], 1u);
}

template <int NT>
__device__ __forceinline__ void topk_rows_row(const size_t row, const float* __restrict__ scores,
                                              int S, int Tn, int K, int q_off,
                                              int32_t* __restrict__ idx,
                                              uint32_t* __restrict__ mask, int mask_stride) {
  __shared__ uint32_t hist[padded(kBins)];
  __shared__ int warp_buf[32];
  __shared__ int scan_total;
  __shared__ uint32_t sel_bin;
  __shared__ int sel_above;
  __shared__ int wgt[NT / 32], weq[NT / 32];

  const int s = (int)(row % (unsigned)S);  // 32-bit: rows < 2^31
  const int n = min(Tn, s + q_off + 1);
  const float* sc = scores + row * (size_t)Tn;
  int32_t* out = idx + row * (size_t)K;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int mwords = mask_stride;  // words per mask row (>= ceil(Tn/32))
  uint32_t* mrow = mask ? mask + row * (size_t)mwords : nullptr;

  if (n <= K) {  // every valid key is kept
    for (int i = tid; i < K; i += NT) out[i] = i < n ? i : -1;
    if (mrow)
      for (int wd = tid; wd < mwords; wd += NT) {
        int lo = wd * 32;
        uint32_t m = lo + 32 <= n ? 0xffffffffu : (lo >= n ? 0u : ((1u << (n - lo)) - 1u));
        mrow[wd] = m;
      }
    return;
  }

  // ---------------- radix select: find the threshold prefix and `need`
  uint32_t prefix = 0;
  int pbits = 0;
  int need = K;
  const int widths[3] = {11, 11, 10};
  for (int pass = 0; pass < 3; ++pass) {
    const int dw = widths[pass];
    const int shift = 32 - pbits - dw;
    for (int i = tid; i < padded(kBins); i += NT) hist[i] = 0;
    __syncthreads();
    for (int i0 = 0; i0 < n; i0 += NT) {
      const int i = i0 + tid;
      uint32_t digit = 0xffffffffu;
      if (i < n) {
        uint32_t key = order_key(sc[i]);
        bool match = pbits == 0 || (key >> (32 - pbits)) == prefix;
        if (match) digit = (key >> shift) & ((1u << dw) - 1u);
      }
      hist_add<NT>(hist, digit, digit != 0xffffffffu);
    }
    __syncthreads();
    // bins from the top: thread j owns a contiguous run of bins, highest first
    constexpr int kPer = kBins / NT;
    const int hi_bin = kBins - tid * kPer;  // exclusive upper end of my run
    int local = 0;
#pragma unroll
    for (int q = 1; q <= kPer; ++q) local += (int)hist[hpad(hi_bin - q)];
    int above = block_excl_scan(local, warp_buf, &scan_total);
#pragma unroll
    for (int q = 1; q <= kPer; ++q) {
      int c = (int)hist[hpad(hi_bin - q)];
      if (above < need && above + c >= need) {
        sel_bin = (uint32_t)(hi_bin - q);
        sel_above = above;
      }
      above += c;
    }
    __syncthreads();
    const uint32_t bsel = sel_bin;
    need -= sel_above;
    prefix = (prefix << dw) | bsel;
    pbits += dw;
    const bool all_taken = (int)hist[hpad(bsel)] == need;
    __syncthreads();
    if (all_taken) break;  // every key in the bucket is kept: no need to refine further
  }

  // ---------------- ordered compaction
  const int fshift = 32 - pbits;
  const uint32_t lt_mask = (1u << lane) - 1u;
  int run_gt = 0, run_eq = 0;
  for (int i0 = 0; i0 < n; i0 += NT) {
    const int i = i0 + tid;
    bool gt = false, eq = false;
    if (i < n) {
      uint32_t hi = order_key(sc[i]) >> fshift;
      gt = hi > prefix;
      eq = hi == prefix;
    }
    const uint32_t bgt = __ballot_sync(0xffffffffu, gt);
    const uint32_t beq = __ballot_sync(0xffffffffu, eq);
    if (lane == 0) {
      wgt[warp] = __popc(bgt);
      weq[warp] = __popc(beq);
    }
    __syncthreads();
    int pg = run_gt, pe = run_eq, tg = 0, te = 0;
#pragma unroll 4
    for (int w2 = 0; w2 < NT / 32; ++w2) {
      int a = wgt[w2], c = weq[w2];
      if (w2 < warp) { pg += a; pe += c; }
      tg += a; te += c;
    }
    const int my_gt = pg + __popc(bgt & lt_mask);
    const int my_eq = pe + __popc(beq & lt_mask);
    const bool sel = gt || (eq && my_eq < need);
    const int pos = my_gt + min(my_eq, need);
    if (sel && pos < K) out[pos] = i;
    if (mrow) {
      const uint32_t bsel = __ballot_sync(0xffffffffu, sel);
      const int wd = (i0 >> 5) + warp;
      if (lane == 0 && wd < mwords) mrow[wd] = bsel;
    }
    run_gt += tg;
    run_eq += te;
    __syncthreads();
  }
  if (mrow) {
    const int written = min(mwords, ((n + NT - 1) / NT) * (NT / 32));
    for (int wd = written + tid; wd < mwords; wd += NT) mrow[wd] = 0u;
  }
}

// One row per CTA iteration over rows blockIdx.x, blockIdx.x + gridDim.x, ...; with run_if,
// nothing happens unless *run_if != 0 (the fused path's fallback).
template <int NT, bool STRIDED>
__global__ void __launch_bounds__(NT) topk_rows_kernel(const float* __restrict__ scores, int S,
                                                       int Tn, int K, int q_off,
                                                       int32_t* __restrict__ idx,
                                                       uint32_t* __restrict__ mask,
                                                       int mask_stride, const int* run_if,
                                                       size_t rows) {
  if (!STRIDED) {
    topk_rows_row<NT>(blockIdx.x, scores, S, Tn, K, q_off, idx, mask, mask_stride);
    return;
  }
  if (*reinterpret_cast<const volatile int*>(run_if) == 0) return;
  for (size_t row = blockIdx.x; row < rows; row += gridDim.x) {
    topk_rows_row<NT>(row, scores, S, Tn, K, q_off, idx, mask, mask_stride);
    __syncthreads();  // shared memory is reused by the next row
  }
}

// ------------------------------------------------------------------------------------
// Two-read top-k with shared-memory bitmaps (rows up to kMaxBitmapKeys keys).
//
// Read 1 (HBM) finds a window of 12-bit buckets (top bits of the order key) that holds the
// K-th key.  Long rows (8192 keys and more) histogram every 8th key and take the buckets
// around the sample's K-th rank (a 3-sigma rank margin); short rows histogram every key and
// the window is the exact bucket b1.  Read 2 (L2, or the registers when the whole row fit in
// read 1's batch of loads): keys above the window go to the SELECTED bitmap, keys inside it
// to the CANDIDATE bitmap -- two float comparisons per key against the window's bucket
// bounds and one warp vote per 32-key word.  The candidates (a few percent of the keys) are
// then listed in shared memory as (key, position) from the bitmap, their scores re-read
// from L2.  On long rows an exact 12-bit histogram of the candidates alone then gives b1;
// if the sampled window missed the K-th key, read 1 is redone exactly.  Either way b1 and
// `need` (keys of b1 still to take) are exact.  The low 20 bits are resolved by two 10-bit
// histogram passes over the candidate list (in shared memory; only a list that overflowed is
// re-read from L2 through the bitmap), giving the exact threshold key tau.  Candidates above tau join SELECTED; candidates equal to tau are
// ranked by index with a prefix scan of their bitmap and the first `need` join SELECTED.
// An ordered scan of SELECTED writes the indices (ascending) and the bitmap itself is the
// selection mask row.
// ------------------------------------------------------------------------------------
constexpr int kMaxBitmapKeys = 1 << 20;
constexpr size_t kMaxDynSmem = 220u * 1024u;  // leaves room for the static shared memory
constexpr int kBins1 = 4096;  // top 12 bits
constexpr int kBins2 = 1024;  // 10-bit refinement digits
static_assert(padded(kBins1) % 4 == 0 && padded(kBins2) % 4 == 0, "clear_words wants x4");

// Bucket holding the need-th largest key: writes (bin, count above it, its count) to
// out[0..2].  Each thread owns a run of NBINS/NT bins, highest first; the counts stay in
// registers across the block scan.
template <int NT, int NBINS>
__device__ __forceinline__ void find_bucket(const uint32_t* hist, int need, int* warp_buf,
                                            int* scan_total, int* out) {
  constexpr int per = NBINS / NT;
  const int hi_bin = NBINS - threadIdx.x * per;
  int c[per];
  int local = 0;
#pragma unroll
  for (int q = 0; q < per; ++q) {
    c[q] = (int)hist[hpad(hi_bin - 1 - q)];
    local += c[q];
  }
  int above = block_excl_scan(local, warp_buf, scan_total);
  if (above < need && above + local >= need) {  // the one thread whose run holds the bin
#pragma unroll
    for (int q = 0; q < per; ++q) {
      if (above < need && above + c[q] >= need) {
        out[0] = hi_bin - 1 - q;
        out[1] = above;
        out[2] = c[q];
      }
      above += c[q];
    }
  }
}

// find_bucket for two ranks need_a <= need_b over one scan: writes the bins holding the
// need_a-th and the need_b-th largest keys to *bin_a, *bin_b (shared; callers pass a barrier
// before reading them).
template <int NT, int NBINS>
__device__ __forceinline__ void find_bucket2(const uint32_t* hist, int need_a, int need_b,
                                             int* warp_buf, int* scan_total, int* bin_a,
                                             int* bin_b) {
  constexpr int per = NBINS / NT;
  const int hi_bin = NBINS - threadIdx.x * per;
  int c[per];
  int local = 0;
#pragma unroll
  for (int q = 0; q < per; ++q) {
    c[q] = (int)hist[hpad(hi_bin - 1 - q)];
    local += c[q];
  }
  int above = block_excl_scan(local, warp_buf, scan_total);
  const bool has_a = above < need_a && above + local >= need_a;
  const bool has_b = above < need_b && above + local >= need_b;
  if (has_a || has_b) {  // only the threads whose runs hold one of the bins
#pragma unroll
    for (int q = 0; q < per; ++q) {
      if (above < need_a && above + c[q] >= need_a) *bin_a = hi_bin - 1 - q;
      if (above < need_b && above + c[q] >= need_b) *bin_b = hi_bin - 1 - q;
      above += c[q];
    }
  }
}

// find_bucket restricted to the bins [lo, hi] (the histogram holds nothing else): the bins
// of a narrow window are scanned by warp 0 alone, highest first; `need` is at most their
// total.  Writes (bin, count above it, its count) to out[0..2]; callers pass a barrier
// before reading them.
template <int NT, int NBINS>
__device__ __forceinline__ void find_bucket_window(const uint32_t* hist, int lo, int hi, int need,
                                                   int* warp_buf, int* scan_total, int* out) {
  if (hi - lo >= 32) {
    find_bucket<NT, NBINS>(hist, need, warp_buf, scan_total, out);
    return;
  }
  if (threadIdx.x >= 32) return;
  const int lane = threadIdx.x, b = hi - lane;
  const int c = b >= lo ? (int)hist[hpad(b)] : 0;
  int x = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  const int above = x - c;
  if (b >= lo && above < need && x >= need) {
    out[0] = b;
    out[1] = above;
    out[2] = c;
  }
}

// Zeroes nwords (a multiple of 4) 32-bit words at a 16-byte aligned address, block-wide.
__device__ __forceinline__ void clear_words(uint32_t* p, int nwords) {
  uint4* q = reinterpret_cast<uint4*>(p);
  for (int i = threadIdx.x; i < nwords / 4; i += blockDim.x) q[i] = make_uint4(0u, 0u, 0u, 0u);
}

// Reserves c consecutive slots per lane in a shared list; returns this lane's first slot.
__device__ __forceinline__ int warp_reserve(int c, int* counter) {
  const int lane = threadIdx.x & 31;
  int x = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  int base = 0;
  if (lane == 31 && x > 0) base = atomicAdd(counter, x);
  base = __shfl_sync(0xffffffffu, base, 31);
  return base + x - c;
}

// U scores per thread, lane-contiguous: slot j of this thread is key base + j*NT + tid, so
// the 32 lanes of a warp hold one 32-key bitmap word per slot.  Keys at or past n load as
// 0.0 (callers mask them).
template <int NT, int U>
__device__ __forceinline__ void load_vals(const float* __restrict__ sc, int n, int base,
                                          float (&v)[U]) {
#pragma unroll
  for (int j = 0; j < U; ++j) {
    const int i = base + j * NT + (int)threadIdx.x;
    v[j] = i < n ? __ldg(sc + i) : 0.f;
  }
}

// The smallest float whose order key lies in bucket b or above (b = 0..4096 over the top 12
// key bits): for every score v that is not NaN, (order_key(v) >> 20) >= b  <=>  v >= this.
// Buckets 0..7 hold only NaN images and, at the top of bucket 7, -inf; bucket 8 starts at
// -FLT_MAX; a bucket past the one of +inf has no float (NaN: no comparison passes).  -0.0 and
// +0.0 share a key and compare equal as floats, so the two tests agree on them as well.
__host__ __device__ __forceinline__ float float_of_bits(uint32_t u) {
  float f;
  memcpy(&f, &u, sizeof f);
  return f;
}
__host__ __device__ __forceinline__ float bucket_floor(uint32_t b) {
  if (b >= 4096u) return float_of_bits(0x7fffffffu);
  const uint32_t k = b << 20;
  if (k < 0x00800000u) return float_of_bits(0xff800000u);         // -inf
  if (k < 0x80000000u) return float_of_bits(~k);                  // a negative float
  const uint32_t u = k ^ 0x80000000u;                             // +0.0 and up
  return u <= 0x7f800000u ? float_of_bits(u) : float_of_bits(0x7fffffffu);
}

// Read 2's vote over one batch of U scores per thread (load_vals layout): slot j of the warp
// is bitmap word (base >> 5) + j * NT/32 + warp; lane 0 stores (keys >= f_hi, keys >= f_lo)
// as one 64-bit pair.  Only a batch that runs past n (FULL false) tests the bounds.
template <int NT, int U, bool FULL>
__device__ __forceinline__ void vote_words(const float (&v)[U], int base, int n, float f_lo,
                                           float f_hi, uint2* bm) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint2* dst = bm + (base >> 5) + warp;
#pragma unroll
  for (int j = 0; j < U; ++j) {
    const int w0 = base + j * NT + warp * 32;  // first key of this warp's word
    bool a = v[j] >= f_hi, b = v[j] >= f_lo;
    if (!FULL) {
      a = a && w0 + lane < n;
      b = b && w0 + lane < n;
    }
    const uint32_t gt = __ballot_sync(0xffffffffu, a);
    const uint32_t ge = __ballot_sync(0xffffffffu, b);
    if (lane == 0 && (FULL || w0 < n)) dst[j * (NT / 32)] = make_uint2(gt, ge);
  }
}

template <int NT, bool SAMPLE>
__device__ __forceinline__ void topk_bitmap_row(const size_t row, const float* __restrict__ scores,
                                                int S, int Tn, int K, int q_off,
                                                int32_t* __restrict__ idx,
                                                uint32_t* __restrict__ mask, int mask_stride,
                                                int cl_cap) {
  extern __shared__ uint32_t dsm[];
  const int W = (Tn + 31) >> 5;              // bitmap words per row
  uint32_t* hist = dsm;                      // [padded(kBins1)]
  // [W] bitmap words: .x SELECTED, .y CANDIDATE (read 2 leaves there the keys at or above
  // the window, collect() removes the SELECTED ones; later the ties at the threshold)
  uint2* bm = reinterpret_cast<uint2*>(hist + padded(kBins1));
  uint32_t* cl_key = reinterpret_cast<uint32_t*>(bm + W);  // [cl_cap] candidate keys
  uint32_t* cl_idx = cl_key + cl_cap;                      // [cl_cap] candidate positions
  __shared__ int warp_buf[32];
  __shared__ int2 warp_buf2[32];
  __shared__ int2 scan_total2;
  __shared__ int scan_total;
  __shared__ int pick[3];
  __shared__ int cnt_sel, cl_n;

  const int s = (int)(row % (unsigned)S);  // 32-bit: rows < 2^31
  const int n = min(Tn, s + q_off + 1);
  const float* sc = scores + row * (size_t)Tn;
  int32_t* out = idx + row * (size_t)K;
  const int tid = threadIdx.x, lane = tid & 31;
  uint32_t* mrow = mask ? mask + row * (size_t)mask_stride : nullptr;
  const int nw = (n + 31) >> 5;

  if (n <= K) {  // every valid key is kept
    for (int i = tid; i < K; i += NT) out[i] = i < n ? i : -1;
    if (mrow)
      for (int wd = tid; wd < mask_stride; wd += NT) {
        const int lo = wd * 32;
        mrow[wd] = lo + 32 <= n ? 0xffffffffu : (lo >= n ? 0u : ((1u << (n - lo)) - 1u));
      }
    return;
  }

  clear_words(hist, padded(kBins1));
  if (tid == 0) { cnt_sel = 0; cl_n = 0; }
  __syncthreads();

  constexpr int U = (NT == 256 && !SAMPLE) ? 16 : 8;  // scores per thread per batch of loads
  constexpr int kChunk = NT * U;                        // keys per batch
  float kv[U];  // the current batch of scores; the whole row when n <= kChunk
  bool held = false;
  uint32_t b1 = 0;
  int need = K, cnt1 = 0;

  // Exact read 1: 12-bit histogram of every key -> bucket b1 of the K-th key, `need`.
  auto exact_read1 = [&]() {
    for (int base = 0; base < n; base += kChunk) {
      load_vals<NT, U>(sc, n, base, kv);
#pragma unroll
      for (int j = 0; j < U; ++j)
        hist_add<NT>(hist, order_key(kv[j]) >> 20, base + j * NT + tid < n);
    }
    held = n <= kChunk;
    __syncthreads();
    find_bucket<NT, kBins1>(hist, K, warp_buf, &scan_total, pick);
    __syncthreads();
    b1 = (uint32_t)pick[0];
    need = K - pick[1];
    cnt1 = pick[2];
  };

  // Read 2: keys whose bucket is above [lo, hi] -> SELECTED bitmap, at or above lo -> the
  // CANDIDATE word (collect() removes the SELECTED keys from it).  The buckets are compared
  // as floats (bucket_floor) and each warp's 32 lanes vote one bitmap word per slot.
  auto read2 = [&](uint32_t lo, uint32_t hi) {
    const float f_lo = bucket_floor(lo), f_hi = bucket_floor(hi + 1u);
    if (held) {
      vote_words<NT, U, false>(kv, 0, n, f_lo, f_hi, bm);
    } else if (SAMPLE) {
      // long rows: two register buffers, the next batch in flight while one is voted
      float vb[U];
      load_vals<NT, U>(sc, n, 0, kv);
      for (int base = 0; base < n; base += 2 * kChunk) {
        if (base + kChunk < n) load_vals<NT, U>(sc, n, base + kChunk, vb);
        if (base + kChunk <= n) vote_words<NT, U, true>(kv, base, n, f_lo, f_hi, bm);
        else vote_words<NT, U, false>(kv, base, n, f_lo, f_hi, bm);
        if (base + kChunk >= n) break;
        if (base + 2 * kChunk < n) load_vals<NT, U>(sc, n, base + 2 * kChunk, kv);
        if (base + 2 * kChunk <= n) vote_words<NT, U, true>(vb, base + kChunk, n, f_lo, f_hi, bm);
        else vote_words<NT, U, false>(vb, base + kChunk, n, f_lo, f_hi, bm);
      }
    } else {
      for (int base = 0; base < n; base += kChunk) {
        load_vals<NT, U>(sc, n, base, kv);
        if (base + kChunk <= n) vote_words<NT, U, true>(kv, base, n, f_lo, f_hi, bm);
        else vote_words<NT, U, false>(kv, base, n, f_lo, f_hi, bm);
      }
    }
    __syncthreads();
  };

  // After read 2: the candidate list (order key, position), built from the CANDIDATE
  // bitmap with the scores re-read from L2, and its length cl_n.  A list longer than cl_cap
  // keeps its first cl_cap entries (cl_n still counts them all); the later steps then walk
  // the bitmap instead.  The sampled window also needs the SELECTED count (cnt_sel) and the
  // 12-bit histogram of the candidates (into `hist`, which is clear).
  auto collect = [&](bool sampled) {
    int lsel = 0;
    for (int w0 = 0; w0 < nw; w0 += NT) {
      const int wd = w0 + tid;
      uint32_t cb = 0u;
      if (wd < nw) {
        const uint2 w = bm[wd];
        if (sampled) lsel += __popc(w.x);
        cb = w.y & ~w.x;
        bm[wd].y = cb;
      }
      int pos = warp_reserve(__popc(cb), &cl_n);
      while (__any_sync(0xffffffffu, cb != 0u)) {
        // two candidates per step, so that two loads are in flight
        int t0 = -1, t1 = -1;
        if (cb) { t0 = wd * 32 + __ffs(cb) - 1; cb &= cb - 1u; }
        if (cb) { t1 = wd * 32 + __ffs(cb) - 1; cb &= cb - 1u; }
        const float v0 = t0 >= 0 ? __ldg(sc + t0) : 0.f;
        const float v1 = t1 >= 0 ? __ldg(sc + t1) : 0.f;
        const uint32_t k0 = order_key(v0), k1 = order_key(v1);
        if (t0 >= 0) {
          if (pos < cl_cap) { cl_key[pos] = k0; cl_idx[pos] = (uint32_t)t0; }
          ++pos;
        }
        if (t1 >= 0) {
          if (pos < cl_cap) { cl_key[pos] = k1; cl_idx[pos] = (uint32_t)t1; }
          ++pos;
        }
        if (sampled) {
          hist_add<NT>(hist, k0 >> 20, t0 >= 0);
          hist_add<NT>(hist, k1 >> 20, t1 >= 0);
        }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) lsel += __shfl_xor_sync(0xffffffffu, lsel, o);
    if (lane == 0 && lsel) atomicAdd(&cnt_sel, lsel);
    __syncthreads();
  };

  if (SAMPLE && n >= 8192) {  // long rows only: on short rows the extra steps cost more
    // ---------------- read 1 (sampled): 12-bit histogram of every 8th key -> a window of
    // buckets that holds the K-th key with high probability (rank margin 3 sigma + 2)
    const int ns = (n + 7) >> 3;
    for (int m0 = 0; m0 < ns; m0 += NT * 8) {
      float v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int m = m0 + u * NT + tid;
        v[u] = m < ns ? __ldg(sc + 8 * m) : 0.f;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) hist_add<NT>(hist, order_key(v[u]) >> 20, m0 + u * NT + tid < ns);
    }
    __syncthreads();
    const float ks = (float)K * (float)ns / (float)n;
    const int delta = (int)(3.0f * sqrtf(ks) + 2.0f);
    const int r_hi = max(1, (int)ks - delta), r_lo = min(ns, (int)ks + delta + 1);
    find_bucket2<NT, kBins1>(hist, r_hi, r_lo, warp_buf, &scan_total, &pick[0], &pick[1]);
    __syncthreads();
    const uint32_t b_hi = (uint32_t)pick[0], b_lo = (uint32_t)pick[1];
    // the candidates fall in the window's bins only: a narrow window clears just those
    if (b_hi - b_lo < 32u) {
      for (int b = (int)b_lo + tid; b <= (int)b_hi; b += NT) hist[hpad(b)] = 0u;
    } else {
      clear_words(hist, padded(kBins1));
    }
    read2(b_lo, b_hi);  // ends with a barrier: the histogram is clear
    collect(true);      // + the SELECTED count and the candidates' 12-bit histogram
    const int nsel = cnt_sel, ncand = cl_n;
    if (nsel < K && nsel + ncand >= K) {
      find_bucket_window<NT, kBins1>(hist, (int)b_lo, (int)b_hi, K - nsel, warp_buf,
                                     &scan_total, pick);
      __syncthreads();
      b1 = (uint32_t)pick[0];
      need = K - nsel - pick[1];
      cnt1 = pick[2];
    } else {
      // the sample missed: exact read 1, then read 2 again with the window [b1, b1]
      __syncthreads();  // every thread has read the counts before they are reset
      clear_words(hist, padded(kBins1));
      if (tid == 0) { cnt_sel = 0; cl_n = 0; }
      __syncthreads();
      exact_read1();
      read2(b1, b1);
      collect(false);
    }
  } else {
    exact_read1();
    read2(b1, b1);
    collect(false);
  }
  const int ncl = cl_n;
  const bool use_cl = ncl <= cl_cap;  // else the candidates are re-read through the bitmap

  // ---------------- refine the low 20 bits over the candidates only
  uint32_t prefix = b1;
  int pbits = 12;
  if (cnt1 != need) {
    for (int pass = 0; pass < 2; ++pass) {
      const int shift = 20 - 10 * (pass + 1);
      clear_words(hist, padded(kBins2));
      __syncthreads();
      if (use_cl) {
        for (int i0 = 0; i0 < ncl; i0 += NT) {
          const int i = i0 + tid;
          uint32_t digit = 0u;
          bool valid = false;
          if (i < ncl) {
            const uint32_t key = cl_key[i];
            if ((key >> (32 - pbits)) == prefix) {
              digit = (key >> shift) & (kBins2 - 1);
              valid = true;
            }
          }
          hist_add<NT>(hist, digit, valid);
        }
      } else {
        for (int w0 = 0; w0 < nw; w0 += NT) {
          const int wd = w0 + tid;
          uint32_t bits = wd < nw ? bm[wd].y : 0u;
          // every lane walks its word; the histogram add is warp-aggregated per step
          bool more = __any_sync(0xffffffffu, bits != 0u);
          while (more) {
            const bool has = bits != 0u;
            uint32_t digit = 0u;
            bool valid = false;
            if (has) {
              const int j = __ffs(bits) - 1;
              bits &= bits - 1u;
              const uint32_t key = order_key(__ldg(sc + wd * 32 + j));
              if ((key >> (32 - pbits)) == prefix) {
                digit = (key >> shift) & (kBins2 - 1);
                valid = true;
              }
            }
            hist_add<NT>(hist, digit, valid);
            more = __any_sync(0xffffffffu, bits != 0u);
          }
        }
      }
      __syncthreads();
      find_bucket<NT, kBins2>(hist, need, warp_buf, &scan_total, pick);
      __syncthreads();
      const uint32_t bsel = (uint32_t)pick[0];
      need -= pick[1];
      prefix = (prefix << 10) | bsel;
      pbits += 10;
      if (pick[2] == need) break;  // every key of the bucket is kept
    }
  }

  // ---------------- candidates: above the threshold -> SELECTED, at it -> ties (CANDIDATE)
  const int fshift = 32 - pbits;
  if (use_cl) {
    for (int wd = tid; wd < nw; wd += NT) bm[wd].y = 0u;
    __syncthreads();
    for (int i = tid; i < ncl; i += NT) {
      const uint32_t hi = cl_key[i] >> fshift, t = cl_idx[i];
      if (hi > prefix) atomicOr(&bm[t >> 5].x, 1u << (t & 31));
      else if (hi == prefix) atomicOr(&bm[t >> 5].y, 1u << (t & 31));
    }
  } else {
    for (int wd = tid; wd < nw; wd += NT) {
      uint32_t bits = bm[wd].y, sel = 0u, tie = 0u;
      while (bits) {
        const int j = __ffs(bits) - 1;
        bits &= bits - 1u;
        const uint32_t hi = order_key(__ldg(sc + wd * 32 + j)) >> fshift;
        if (hi > prefix) sel |= 1u << j;
        else if (hi == prefix) tie |= 1u << j;
      }
      bm[wd].x |= sel;
      bm[wd].y = tie;
    }
  }
  __syncthreads();
  // Ordered output.  Thread t owns words [t*per, t*per+per); one scan gives, per thread, the
  // selected keys and the ties before its words.  Ties are ranked by index: the first `need`
  // are kept, so a thread keeps its first max(0, min(ties, need - ties before)) ties, and
  // its first output slot is (selected before) + min(ties before, need).  The mask row gets
  // the same words.
  const int per = (nw + NT - 1) / NT;
  {
    int lsel = 0, ltie = 0;
    for (int q = 0; q < per; ++q) {
      const int wd = tid * per + q;
      if (wd < nw) {
        const uint2 w = bm[wd];
        lsel += __popc(w.x);
        ltie += __popc(w.y);
      }
    }
    int sel_before, tie_before, sel_total, tie_total;
    block_excl_scan2(lsel, ltie, warp_buf2, &scan_total2, &sel_before, &tie_before, &sel_total,
                     &tie_total);
    const int kneed = max(need, 0);
    int keep = max(0, min(ltie, kneed - tie_before));
    int pos = sel_before + min(tie_before, kneed);
    for (int q = 0; q < per; ++q) {
      const int wd = tid * per + q;
      if (wd >= nw) break;
      uint32_t tb = bm[wd].y, kept = 0u;
      while (tb && keep > 0) {
        const uint32_t low = tb & (0u - tb);
        kept |= low;
        tb ^= low;
        --keep;
      }
      uint32_t bits = bm[wd].x | kept;
      if (mrow) mrow[wd] = bits;
      while (bits) {
        const int j = __ffs(bits) - 1;
        bits &= bits - 1u;
        if (pos < K) out[pos] = wd * 32 + j;
        ++pos;
      }
    }
    const int total = sel_total + min(tie_total, kneed);
    for (int i = total + tid; i < K; i += NT) out[i] = -1;  // only if something went wrong
  }
  if (mrow)
    for (int wd = nw + tid; wd < mask_stride; wd += NT) mrow[wd] = 0u;
}


// Register caps keep 5 (256-thread) or 3 (512-thread) rows in flight per SM.  One row per
// CTA; the STRIDED form (the fused path's fallback) takes rows blockIdx.x, blockIdx.x +
// gridDim.x, ... and does nothing unless *run_if != 0.
template <int NT, bool SAMPLE, bool STRIDED>
__global__ void __launch_bounds__(NT, NT == 256 ? 5 : (NT == 512 ? 3 : 1))
    topk_bitmap_kernel(const float* __restrict__ scores, int S, int Tn, int K, int q_off,
                       int32_t* __restrict__ idx, uint32_t* __restrict__ mask, int mask_stride,
                       int cl_cap, const int* run_if, size_t rows) {
  if (!STRIDED) {
    topk_bitmap_row<NT, SAMPLE>(blockIdx.x, scores, S, Tn, K, q_off, idx, mask, mask_stride,
                                cl_cap);
    return;
  }
  if (*reinterpret_cast<const volatile int*>(run_if) == 0) return;
  for (size_t row = blockIdx.x; row < rows; row += gridDim.x) {
    topk_bitmap_row<NT, SAMPLE>(row, scores, S, Tn, K, q_off, idx, mask, mask_stride, cl_cap);
    __syncthreads();  // shared memory is reused by the next row
  }
}

// ------------------------------------------------------------------------------------
// Fused indexer -> top-k: the threshold and the exact select over candidates.
//
// The top-k of a row only depends on its keys whose score is at least the row's K-th
// largest score tau*.  If a threshold tau <= tau* is known before the row's scores exist,
// the indexer can keep only the keys with score >= tau (its candidates) instead of writing
// every score: when at least K keys pass, tau* >= tau, so every key of the top-k -- and
// every key tied with the K-th -- is a candidate, and the exact select over the candidates
// (same order: higher score, then lower index) is the top-k of the row.
//
// tau comes from a sample: the indexer first scores every kstride-th key tile of each row;
// tau is the r-th largest sampled score, with r the expected sample rank of the K-th key
// (K * n_s / n) plus a six-sigma binomial margin.  Rows with at most `cap` causal keys keep
// every key (tau = the smallest order key).  Whether the sample was right is checked, not
// assumed: a row with fewer than K candidates (tau too high) or more than `cap` (the list
// overflowed) raises a flag, and the stream then runs the full-score indexer and top-k over
// the whole launch, so the result is the same in every case.
// ------------------------------------------------------------------------------------

// Sample keys of a row with last causal key t_last: tiles j = 0..jmax at positions
// j*kstride*128 (all full but the last).
__device__ __forceinline__ int sample_keys(int t_last, int kstride, int* jmax) {
  const int jm = (t_last / 128) / kstride;
  *jmax = jm;
  return jm * 128 + min(128, t_last + 1 - jm * kstride * 128);
}

// tau[row]: the order key of the r-th largest sampled score of the row (radix select on
// the order keys, digits of 11, 11 and 10 bits; an early stop keeps the bucket's smallest
// key, which is <= the r-th largest, so the threshold stays conservative).
template <int NT>
__global__ void __launch_bounds__(NT) topk_tau_kernel(const float* __restrict__ sample,
                                                      long long ld, int S, int Tn, int K,
                                                      int q_off, int kstride, int cap,
                                                      uint32_t* __restrict__ tau) {
  extern __shared__ uint32_t row_keys[];  // [ld] order keys of the sampled row
  __shared__ uint32_t hist[padded(kBins)];
  __shared__ int warp_buf[32];
  __shared__ int scan_total;
  __shared__ uint32_t sel_bin;
  __shared__ int sel_above;
  const size_t row = blockIdx.x;
  const int s = (int)(blockIdx.x % (unsigned)S);
  const int t_last = min(Tn - 1, s + q_off);
  const int n = t_last + 1;
  const int tid = threadIdx.x;
  if (n <= cap) {  // the whole row fits the candidate list: keep every key
    if (tid == 0) tau[row] = 0u;
    return;
  }
  int jmax;
  const int ns = sample_keys(t_last, kstride, &jmax);
  const int m = (jmax + 1) * 128;  // sampled columns of this row
  const float mu = (float)K * (float)ns / (float)n;
  const int r = min(ns, (int)ceilf(mu + 6.0f * sqrtf(mu) + 8.0f));
  const float* sc = sample + row * (size_t)ld;
  // the row's sampled keys, read once: column i holds key (i / 128) * kstride * 128 + i % 128;
  // columns past the row's last causal key (-inf, or never written when they lie past T)
  // become key 0, below every real score's key, and are not counted
  for (int i = tid; i < m; i += NT)
    row_keys[i] = (i >> 7) * kstride * 128 + (i & 127) > t_last ? 0u : order_key(__ldg(sc + i));
  uint32_t prefix = 0;
  int pbits = 0, need = r;
  const int widths[3] = {11, 11, 10};
  for (int pass = 0; pass < 3; ++pass) {
    const int dw = widths[pass];
    const int shift = 32 - pbits - dw;
    for (int i = tid; i < padded(kBins); i += NT) hist[i] = 0;
    __syncthreads();
    for (int i = tid; i < m; i += NT) {
      const uint32_t key = row_keys[i];
      if (key == 0u) continue;  // not a sampled causal key
      const bool match = pbits == 0 || (key >> (32 - pbits)) == prefix;
      hist_add<NT>(hist, (key >> shift) & ((1u << dw) - 1u), match);
    }
    __syncthreads();
    constexpr int kPer = kBins / NT;
    const int hi_bin = kBins - tid * kPer;
    int local = 0;
#pragma unroll
    for (int q = 1; q <= kPer; ++q) local += (int)hist[hpad(hi_bin - q)];
    int above = block_excl_scan(local, warp_buf, &scan_total);
#pragma unroll
    for (int q = 1; q <= kPer; ++q) {
      const int c = (int)hist[hpad(hi_bin - q)];
      if (above < need && above + c >= need) {
        sel_bin = (uint32_t)(hi_bin - q);
        sel_above = above;
      }
      above += c;
    }
    __syncthreads();
    const uint32_t bsel = sel_bin;
    need -= sel_above;
    prefix = (prefix << dw) | bsel;
    pbits += dw;
    const bool all_taken = (int)hist[hpad(bsel)] == need;
    __syncthreads();
    if (all_taken) break;
  }
  if (tid == 0) tau[row] = pbits == 32 ? prefix : prefix << (32 - pbits);
}

// The exact top-k of a row from its candidate list (order key, key index; unordered), or
// the fallback flag when the list cannot hold it.  Output as topk_bitmap_kernel: ascending
// indices, -1 padding, and the selection bitmask.
template <int NT>
__global__ void __launch_bounds__(NT) topk_candidates_kernel(
    const uint2* __restrict__ cand, const int* __restrict__ cand_cnt, int cap, int S, int Tn,
    int K, int q_off,
    int32_t* __restrict__ idx, uint32_t* __restrict__ mask, int mask_stride,
    int* __restrict__ fail) {
  extern __shared__ uint32_t dsm[];
  __shared__ int warp_buf[32];
  __shared__ int scan_total;
  __shared__ uint32_t sel_bin;
  __shared__ int sel_above;
  const size_t row = blockIdx.x;
  const int s = (int)(blockIdx.x % (unsigned)S);
  const int n = min(Tn, s + q_off + 1);
  const int tid = threadIdx.x;
  int32_t* out = idx + row * (size_t)K;
  uint32_t* mrow = mask ? mask + row * (size_t)mask_stride : nullptr;
  if (n <= K) {  // every valid key is kept
    for (int i = tid; i < K; i += NT) out[i] = i < n ? i : -1;
    if (mrow)
      for (int wd = tid; wd < mask_stride; wd += NT) {
        const int lo = wd * 32;
        mrow[wd] = lo + 32 <= n ? 0xffffffffu : (lo >= n ? 0u : ((1u << (n - lo)) - 1u));
      }
    return;
  }
  const int m = __ldg(cand_cnt + row);
  if (m < K || m > cap) {  // the threshold missed (too high) or the list overflowed
    if (tid == 0) atomicExch(fail, 1);
    return;
  }
  const int nw = (n + 31) >> 5;
  uint32_t* hist = dsm;                     // [padded(kBins)]
  uint32_t* ck = hist + padded(kBins);      // [cap]
  uint32_t* ct = ck + cap;                  // [cap]
  uint32_t* selb = ct + cap;                // [nw]
  uint32_t* tieb = selb + nw;               // [nw]
  const uint2* gc = cand + row * (size_t)cap;
  for (int i = tid; i < m; i += NT) {
    const uint2 c = __ldg(gc + i);
    ck[i] = c.x;
    ct[i] = c.y;
  }
  for (int wd = tid; wd < nw; wd += NT) { selb[wd] = 0u; tieb[wd] = 0u; }
  // ---------------- radix select of the K-th largest candidate key
  uint32_t prefix = 0;
  int pbits = 0, need = K;
  const int widths[3] = {11, 11, 10};
  for (int pass = 0; pass < 3; ++pass) {
    const int dw = widths[pass];
    const int shift = 32 - pbits - dw;
    for (int i = tid; i < padded(kBins); i += NT) hist[i] = 0;
    __syncthreads();
    for (int i = tid; i < m; i += NT) {
      const uint32_t key = ck[i];
      const bool match = pbits == 0 || (key >> (32 - pbits)) == prefix;
      hist_add<NT>(hist, (key >> shift) & ((1u << dw) - 1u), match);
    }
    __syncthreads();
    constexpr int kPer = kBins / NT;
    const int hi_bin = kBins - tid * kPer;
    int local = 0;
#pragma unroll
    for (int q = 1; q <= kPer; ++q) local += (int)hist[hpad(hi_bin - q)];
    int above = block_excl_scan(local, warp_buf, &scan_total);
#pragma unroll
    for (int q = 1; q <= kPer; ++q) {
      const int c = (int)hist[hpad(hi_bin - q)];
      if (above < need && above + c >= need) {
        sel_bin = (uint32_t)(hi_bin - q);
        sel_above = above;
      }
      above += c;
    }
    __syncthreads();
    const uint32_t bsel = sel_bin;
    need -= sel_above;
    prefix = (prefix << dw) | bsel;
    pbits += dw;
    const bool all_taken = (int)hist[hpad(bsel)] == need;
    __syncthreads();
    if (all_taken) break;
  }
  // ---------------- above the threshold -> SELECTED, at it -> ties
  const int fshift = 32 - pbits;
  for (int i = tid; i < m; i += NT) {
    const uint32_t hi = ck[i] >> fshift, t = ct[i];
    if (hi > prefix) atomicOr(&selb[t >> 5], 1u << (t & 31));
    else if (hi == prefix) atomicOr(&tieb[t >> 5], 1u << (t & 31));
  }
  __syncthreads();
  // ties ranked by index: the first `need` are kept.  Thread t owns words [t*per, t*per+per).
  const int per = (nw + NT - 1) / NT;
  {
    int local = 0;
    for (int q = 0; q < per; ++q) {
      const int wd = tid * per + q;
      if (wd < nw) local += __popc(tieb[wd]);
    }
    int rank = block_excl_scan(local, warp_buf, &scan_total);
    for (int q = 0; q < per && rank < need; ++q) {
      const int wd = tid * per + q;
      if (wd >= nw) break;
      uint32_t bits = tieb[wd];
      while (bits && rank < need) {
        const int j = __ffs(bits) - 1;
        bits &= bits - 1u;
        selb[wd] |= 1u << j;
        ++rank;
      }
    }
  }
  __syncthreads();
  // ---------------- ordered output: prefix popcounts of SELECTED
  {
    int local = 0;
    for (int q = 0; q < per; ++q) {
      const int wd = tid * per + q;
      if (wd < nw) local += __popc(selb[wd]);
    }
    int pos = block_excl_scan(local, warp_buf, &scan_total);
    for (int q = 0; q < per; ++q) {
      const int wd = tid * per + q;
      if (wd >= nw) break;
      uint32_t bits = selb[wd];
      while (bits) {
        const int j = __ffs(bits) - 1;
        bits &= bits - 1u;
        if (pos < K) out[pos] = wd * 32 + j;
        ++pos;
      }
    }
    const int total = scan_total;
    for (int i = total + tid; i < K; i += NT) out[i] = -1;
  }
  if (mrow)
    for (int wd = tid; wd < mask_stride; wd += NT) mrow[wd] = wd < nw ? selb[wd] : 0u;
}

// Selection bitmask from index lists: bit t of row (b,s) is set when t appears in the row,
// 0 <= t < T and t <= s + q_off (the causal mask).  One CTA per row.
__global__ void idx_to_mask_kernel(const int32_t* __restrict__ idx, int S, int Tn, int K,
                                   int q_off, uint32_t* __restrict__ mask, int stride) {
  const size_t row = blockIdx.x;
  const int spos = (int)(blockIdx.x % (unsigned)S) + q_off;
  uint32_t* m = mask + row * (size_t)stride;
  for (int w = threadIdx.x; w < stride; w += blockDim.x) m[w] = 0u;
  __syncthreads();
  const int32_t* ir = idx + row * (size_t)K;
  for (int i = threadIdx.x; i < K; i += blockDim.x) {
    const int t = ir[i];
    if (t >= 0 && t < Tn && t <= spos) atomicOr(&m[t >> 5], 1u << (t & 31));
  }
}

}  // namespace

cudaError_t launch_idx_to_mask(const int32_t* idx, int B, int S, int T, int K, int q_off,
                               uint32_t* mask, int mask_stride, cudaStream_t st) {
  const size_t rows = (size_t)B * S;
  if (rows == 0) return cudaSuccess;
  idx_to_mask_kernel<<<(unsigned)rows, 256, 0, st>>>(idx, S, T, K, q_off, mask, mask_stride);
  return cudaGetLastError();
}

// The bitmap top-k with its dynamic shared memory: one CTA per row, or (strided) the fused
// path's fallback form.
template <int NT, bool SAMPLE>
cudaError_t launch_bitmap(bool strided, unsigned grid, size_t smem, cudaStream_t st,
                          const float* scores, int S, int T, int K, int q_off, int32_t* idx,
                          uint32_t* mask, int mask_stride, int cap, const int* run_if,
                          size_t rows) {
  auto kern = strided ? topk_bitmap_kernel<NT, SAMPLE, true>
                      : topk_bitmap_kernel<NT, SAMPLE, false>;
  // dynamic + static shared memory may pass the 48 KB default
  cudaError_t e =
      cudaFuncSetAttribute((const void*)kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<grid, NT, smem, st>>>(scores, S, T, K, q_off, idx, mask, mask_stride, cap, run_if, rows);
  return cudaGetLastError();
}

cudaError_t launch_topk_tau(const float* sample, long long ld, int B, int S, int T, int K,
                            int q_off, int kstride, int cap, uint32_t* tau, cudaStream_t st) {
  const size_t rows = (size_t)B * S;
  if (rows == 0) return cudaSuccess;
  const size_t smem = (size_t)ld * sizeof(uint32_t);
  if (smem > kMaxDynSmem) return cudaErrorNotSupported;
  cudaError_t e = cudaFuncSetAttribute((const void*)topk_tau_kernel<256>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  topk_tau_kernel<256><<<(unsigned)rows, 256, smem, st>>>(sample, ld, S, T, K, q_off, kstride,
                                                          cap, tau);
  return cudaGetLastError();
}

size_t topk_candidates_smem(int T, int cap) {
  const int W = (T + 31) / 32;
  return (size_t)(padded(kBins) + 2 * cap + 2 * W) * sizeof(uint32_t);
}

cudaError_t launch_topk_candidates(const uint2* cand, const int* cand_cnt, int cap, int B,
                                   int S, int T, int K,
                                   int q_off, int32_t* idx, uint32_t* mask, int mask_stride,
                                   int* fail, cudaStream_t st) {
  const size_t rows = (size_t)B * S;
  if (rows == 0) return cudaSuccess;
  if (mask && mask_stride < (T + 31) / 32) return cudaErrorInvalidValue;
  const size_t smem = topk_candidates_smem(T, cap);
  if (smem > kMaxDynSmem) return cudaErrorNotSupported;
  cudaError_t e = cudaFuncSetAttribute((const void*)topk_candidates_kernel<256>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  topk_candidates_kernel<256><<<(unsigned)rows, 256, smem, st>>>(
      cand, cand_cnt, cap, S, T, K, q_off, idx, mask, mask_stride, fail);
  return cudaGetLastError();
}

float topk_bucket_floor(unsigned b) { return bucket_floor(b); }

cudaError_t launch_topk(const float* scores, int B, int S, int T, int K, int q_off,
                        int32_t* idx, uint32_t* mask, int mask_stride, cudaStream_t st,
                        const int* run_if) {
  const size_t rows = (size_t)B * S;
  if (rows == 0) return cudaSuccess;
  // one CTA per row; a fallback launch (run_if) takes a grid of a few CTAs per SM that loop
  // over the rows, so that it costs almost nothing when it has nothing to do
  const unsigned grid = (unsigned)(run_if ? (rows < 148u * 4u ? rows : 148u * 4u) : rows);
  if (mask && mask_stride < (T + 31) / 32) return cudaErrorInvalidValue;
  // Bitmap kernel while its shared memory fits: the 4096-bin histogram, two bitmaps of the
  // row and a candidate list (1024 entries for short rows, 2048 for long ones, 512 when
  // the bitmaps are large; the list overflowing only costs re-reads through the bitmap).
  const int W = (T + 31) / 32;
  int cap = T > 8192 ? 2048 : 1024;
  auto smem_for = [&](int c) {
    return (size_t)(padded(kBins1) + 2 * W + 2 * c) * sizeof(uint32_t);
  };
  if (smem_for(cap) > kMaxDynSmem) cap = 512;
  if (T <= kMaxBitmapKeys && smem_for(cap) <= kMaxDynSmem) {
    // one CTA per row; small CTAs so that several rows are in flight per SM (each row is a
    // chain of dependent reads and block-wide scans)
    const size_t smem = smem_for(cap);
    const bool strided = run_if != nullptr;
    if (rows < 296 && T > 8192)  // few long rows (decode): the widest CTA per row
      return launch_bitmap<1024, true>(strided, grid, smem, st, scores, S, T, K, q_off, idx, mask,
                                       mask_stride, cap, run_if, rows);
    // long rows: 256-thread CTAs while five of them fit an SM's shared memory (more rows in
    // flight for the per-row steps between barriers: 32768-key rows 6% faster), else 512
    // (at 65536 keys only four 256-thread rows would fit: 18% slower)
    if (T > 8192 && smem <= 45u * 1024u)
      return launch_bitmap<256, true>(strided, grid, smem, st, scores, S, T, K, q_off, idx, mask,
                                      mask_stride, cap, run_if, rows);
    if (T > 8192)
      return launch_bitmap<512, true>(strided, grid, smem, st, scores, S, T, K, q_off, idx, mask,
                                      mask_stride, cap, run_if, rows);
    return launch_bitmap<256, false>(strided, grid, smem, st, scores, S, T, K, q_off, idx, mask,
                                     mask_stride, cap, run_if, rows);
  }
  const int nt = T >= 8192 ? 1024 : (T >= 2048 ? 512 : 256);
  auto kern = nt == 1024 ? (run_if ? topk_rows_kernel<1024, true> : topk_rows_kernel<1024, false>)
            : nt == 512  ? (run_if ? topk_rows_kernel<512, true> : topk_rows_kernel<512, false>)
                         : (run_if ? topk_rows_kernel<256, true> : topk_rows_kernel<256, false>);
  kern<<<grid, nt, 0, st>>>(scores, S, T, K, q_off, idx, mask, mask_stride, run_if, rows);
  return cudaGetLastError();
}

}  // namespace dsa
