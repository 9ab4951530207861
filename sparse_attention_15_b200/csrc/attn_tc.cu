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
// double-buffered so S_{j+1} = Q K_{j+1}^T overlaps the softmax of block j), O0, O1 (Dv
// columns each, one per softmax group);
// P is split into bf16 P_hi + P_lo (two per 32-bit column): the 16 keys of each chunk write
// P_hi into the first 8 of their own 16 S columns and P_lo into the next 8, which feed
// O += P_hi V + P_lo V as tensor-memory A operands -- the low part keeps the float32
// probabilities' precision that a single bf16 P would lose.  The running max is only raised
// (and O, l rescaled) when a row's block max exceeds it by more than 2^8, so exp2 arguments
// stay <= 8 and rescales are rare.
//
// Roles (16 warps, a setmaxnreg split per warpgroup): warps 0..7 softmax in two groups that
// take alternate key blocks (thread = query row = TMEM lane), each with its own O accumulator
// and running (max, sum); warp 8 TMA producer of Q and K, warp 10 of V, warp 9 the MMA issuer
// (one thread); warps 12..15 merge the two groups' O at the end of an item, normalise, gate
// and store it while the softmax groups start the next item.  Band items, a few key blocks
// long, run one softmax group of all eight warps over every block instead -- two threads per
// row, half of the block's keys each, one O -- and store their output themselves.  Key blocks come from a per-query-block list of the blocks that hold a
// selected key.  Persistent CTAs take items in snake order, longest first (in bands of query
// blocks when K/V exceeds the L2).  Every wait is bounded.
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace dsa {

namespace {

constexpr int kBlk = 128;     // queries per item = keys per block
// Warp roles: 0..7 softmax (two groups of four: warp % 4 is the TMEM lane quadrant),
// 8 TMA producer of Q and K, 9 MMA issuer (and TMEM owner), 10 TMA producer of V (warp 11
// only completes that warpgroup), 12..15 the output epilogue of each item (one thread per
// query row): the softmax groups hand over their (m, l) and go on to the next item while
// the epilogue reads O out.  In band mode (items of a few key blocks, whose epilogue is on
// the path to the next item's first P V) the eight softmax warps form one group (warp / 4
// picks the half of each block's keys) and write the output themselves, each half of the
// columns, and warps 12..15 idle.
constexpr int kSoftWarps = 8;
constexpr int kWarpQK = 8, kWarpMma = 9, kWarpV = 10;
constexpr int kEpiWarp0 = 12;
// Register split (setmaxnreg, per warpgroup, FaCfg::REGS_*): the CTA is launched with 512
// threads x 128 registers = 65536; the two softmax warpgroups raise theirs and the control and
// epilogue warpgroups lower theirs.
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
  int nsink;             // attention sinks (PAS), 0..128: one extra block per item
  // the key blocks each 128-query block visits (mask mode; NULL: every causal block):
  // bcount[b*nqb+qb] of them, in ascending order in blist[(b*nqb+qb)*nkb ...]
  const int* bcount;
  const uint16_t* blist;
  int nkb;
  int band;              // item order: 0 = heads fastest, > 0 = bands of query blocks
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
  static constexpr int BAR_BYTES = BAND ? 512 : 256;
  static constexpr int ML_BYTES = 2 * 2 * kBlk * 2 * 4;  // [buffer][group or half][row][m,l]
  static constexpr int XCH_BYTES = BAND ? 2 * 2 * kBlk * 4 : 0;  // [block parity][half][row]
  static constexpr int SMEM =
      Q_BYTES + STAGES * KV_BYTES + BAR_BYTES + ML_BYTES + XCH_BYTES + 1024;
  // softmax rows of 128 keys (selection form) need 192 registers, half rows (band form) 160
  static constexpr int REGS_SOFT = BAND ? 160 : 192, REGS_CTL = BAND ? 96 : 64,
                       REGS_EPI = BAND ? 96 : 64;
  static_assert(2 * 128 * REGS_SOFT + 128 * REGS_CTL + 128 * REGS_EPI <= 512 * 128,
                "register split");
  static constexpr int THREADS = 32 * 16;
  static constexpr int S_COLS = kBlk;              // fp32 columns of one S buffer
  static constexpr int O_COL = 2 * S_COLS;         // O0, O1 (band: one O) after S0, S1
  static constexpr int TMEM_COLS = 512;
  static_assert(DQK % 64 == 0 && DV % 64 == 0 && DV <= 128, "head dims");
  static_assert(O_COL + 2 * DV <= TMEM_COLS, "TMEM budget");
};

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int x, int y,
                                            int z, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
      "l"(map), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
      : "memory");
}

// Item i -> (query block, batch row, head), longest query blocks first.  When every head's
// K/V fits in L2 the heads vary fastest (a plain longest-first order, which balances the
// CTAs best).  Otherwise (band > 0) the query blocks go in bands of `band` blocks, longest
// band first, and within a band head by head: the CTAs working at the same time then walk
// the key blocks of a few heads, whose K/V stays in L2 while they share it, instead of
// every head's K/V at once; the lengths inside a band differ by at most `band` blocks.
struct Item {
  int qb, b, h;
};
// The k-th item of CTA c: items are dealt in snake order (0..G-1, then G-1..0, ...), so a CTA
// that took one of the longest causal items in a round takes one of the shorter in the next.
__device__ __forceinline__ int snake_item(int k, int c, int G) {
  return k * G + ((k & 1) ? (G - 1 - c) : c);
}
// Items over `nq` query blocks per (batch row, head), in the order above.
__device__ __forceinline__ Item order_item(int i, int H, int B, int nq, int band) {
  Item it;
  if (band <= 0) {
    it.h = i % H;
    const int r = i / H;
    it.b = r % B;
    it.qb = nq - 1 - r / B;
    return it;
  }
  const int per_band = band * B * H;  // items of one full band
  const int bi = i / per_band;        // band index (longest first)
  const int r0 = i - bi * per_band;
  const int q0 = bi * band;           // first (reversed) query block of the band
  const int nb = min(band, nq - q0);  // blocks in this band (the last may be short)
  const int per_head = nb * B;
  it.h = r0 / per_head;
  const int r = r0 - it.h * per_head;
  it.b = r % B;
  it.qb = nq - 1 - (q0 + r / B);
  return it;
}
__device__ __forceinline__ Item item_of(const AttnArgs& a, int i) {
  return order_item(i, a.H, a.B, a.nqb, a.band);
}
// Key blocks [j0, j1) item `it` must visit.  With attention sinks an item first visits one
// sink block (the nsink sink entries, always visible), then those key blocks: block r of
// the item is the sink block for r < sink_blocks(a), else key block j0 + r - sink_blocks.
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

template <bool BAND>
__device__ __forceinline__ int sink_blocks(const AttnArgs& a) {
  return a.nsink > 0 ? 1 : 0;
}

// Empty tiles are skipped ([AXK2] "注意力前向的骨架": under the additive sparse mask a key block
// no query of the item selected contributes exp(-inf) = 0 to every row): with a block list
// an item visits only the key blocks some query of its 128-query block selected from, in
// ascending order (a block with no selection at all still gets one block, key block 0, so
// that every item has one and its outputs -- zeros -- are written by the same path).
struct KeyBlocks {
  const uint16_t* list;  // the item's key blocks, or NULL: every block of [j0, j1)
  int n, j0;
  __device__ __forceinline__ int at(int r) const { return list ? (int)__ldg(list + r) : j0 + r; }
};

__device__ __forceinline__ KeyBlocks key_blocks(const AttnArgs& a, const Item& it, int j0,
                                                int j1) {
  KeyBlocks kb;
  kb.j0 = j0;
  if (a.blist) {
    const size_t q = (size_t)it.b * a.nqb + it.qb;
    kb.list = a.blist + q * a.nkb;
    kb.n = __ldg(a.bcount + q);
  } else {
    kb.list = nullptr;
    kb.n = j1 - j0;
  }
  return kb;
}

template <class C>
__global__ void __launch_bounds__(C::THREADS, 1)
    masked_attn_tc_kernel(const __grid_constant__ CUtensorMap qmap,
                          const __grid_constant__ CUtensorMap kmap,
                          const __grid_constant__ CUtensorMap vmap,
                          const __grid_constant__ CUtensorMap skmap,
                          const __grid_constant__ CUtensorMap svmap, const AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* Qs = smem;
  uint8_t* KVs = smem + C::Q_BYTES;  // [STAGES] x (K block, V block)
  uint64_t* bars = reinterpret_cast<uint64_t*>(KVs + C::STAGES * C::KV_BYTES);
  uint64_t* q_full = bars;           // 1
  uint64_t* q_empty = bars + 1;      // 1
  uint64_t* k_full = bars + 2;       // [2] K block landed
  // bars + 4, + 5: unused (a K stage is free once s_full of its block completes)
  uint64_t* s_full = bars + 6;       // [2]
  uint64_t* p_full = bars + 10;      // [2]
  uint64_t* pv_done = bars + 12;     // [2] (one phase per block of that parity)
  uint64_t* o_empty = bars + 14;     // 1 (one phase per item)
  uint64_t* mma_done = bars + 16;    // 1
  uint64_t* v_full = bars + 17;      // [2] V block landed
  // bars + 19, + 20: unused (a V stage is free once pv_done of its block completes)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 21);
  uint64_t* ml_full = bars + 22;     // [2] (m, l) of item ni in buffer ni & 1 written
  uint64_t* ml_empty = bars + 24;    // [2] ... and read by the epilogue
  // band: [4 quadrants][2 block parities], the two softmax halves of a quadrant meet per block
  uint64_t* xbar = bars + 32;
  float* ml = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(bars) + C::BAR_BYTES);
  float* xch = ml + C::ML_BYTES / 4;  // band: the two halves' block maxima of each row

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_items = a.B * a.H * a.nqb;
  const int group = a.H / a.HKV;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1); mbar_init(q_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], C::BAND ? 8 : 4);  // the band's one group has eight warps
    }
    mbar_init(&pv_done[0], 1); mbar_init(&pv_done[1], 1);
    // o_empty: the four epilogue warps, or in band mode the eight softmax warps
    mbar_init(o_empty, C::BAND ? 8 : 4); mbar_init(mma_done, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&ml_full[i], 8 * 32);
      mbar_init(&ml_empty[i], 4 * 32);
    }
    if (C::BAND)
      for (int i = 0; i < 8; ++i) mbar_init(&xbar[i], 64);
    fence_mbar_init();
    prefetch_tmap(&qmap); prefetch_tmap(&kmap); prefetch_tmap(&vmap);
    if (sink_blocks<C::BAND>(a)) { prefetch_tmap(&skmap); prefetch_tmap(&svmap); }
  }
  if (warp == kWarpMma) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp >= kSoftWarps && warp < kEpiWarp0) {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::REGS_CTL));
  if (warp == kWarpQK || warp == kWarpV) {
    // ------------------------------------------------------------------ TMA producers
    // warp 0: Q blocks and K blocks; warp 2: V blocks.  K and V have separate rings: a K
    // stage is free as soon as S = Q K^T is done, long before the P V of the same block, so
    // the next K blocks stream in while the softmax runs.  The MMA thread's commits for the
    // softmax (s_full) and for the end of P V (pv_done) free the stages as well: block g of
    // a ring waits for the phase of block g - 2, and neither barrier can run further ahead,
    // since block g's own product needs the copy this thread is about to start.
    const bool kq = warp == kWarpQK;
    if (lane == 0) {
      uint32_t g = 0, ni = 0;
      bool ok = true;
      uint64_t* full = kq ? k_full : v_full;
      uint64_t* empty = kq ? s_full : pv_done;
      for (int kk_ = 0, i = snake_item(0, blockIdx.x, gridDim.x); ok && i < n_items;
           i = snake_item(++kk_, blockIdx.x, gridDim.x), ++ni) {
        const Item it = item_of(a, i);
        int j0, j1;
        key_range<C::BAND>(a, it, &j0, &j1);
        if (kq) {
          if (ni > 0 && !mbar_wait(q_empty, (ni - 1) & 1)) { ok = false; break; }
          mbar_arrive_expect_tx(q_full, C::Q_BYTES);
          const int qrow = it.b * a.S + it.qb * kBlk;
#pragma unroll
          for (int x = 0; x < C::QKH; ++x)
            tma_load_3d(Qs + x * C::SLICE, &qmap, x * 64, it.h, qrow, q_full);
        }
        const int kvh = it.h / group;
        const int sb = sink_blocks<C::BAND>(a);
        const KeyBlocks kb = key_blocks(a, it, j0, j1);
        const int nb = kb.n + sb;
        // key block of position r, read from the block list one position ahead
        int blk_next = nb > sb ? kb.at(0) : 0;
        for (int r = 0; r < nb; ++r, ++g) {
          const int st = g & 1;
          // the sink block reads rows 0..127 of the sink arrays (rows past nsink: zero fill)
          const bool sink = r < sb;
          int blk = 0;
          if (!sink) {
            blk = blk_next;
            if (r + 1 < nb) blk_next = kb.at(r + 1 - sb);
          }
          if (g >= 2 && !mbar_wait(&empty[st], ((g >> 1) - 1) & 1)) { ok = false; break; }
          uint8_t* dst = KVs + st * C::KV_BYTES + (kq ? 0 : C::K_BYTES);
          const int krow = sink ? 0 : it.b * a.T + blk * kBlk;
          if (kq) {
            mbar_arrive_expect_tx(&full[st], C::K_BYTES);
#pragma unroll
            for (int x = 0; x < C::QKH; ++x)
              tma_load_3d(dst + x * C::SLICE, sink ? &skmap : &kmap, x * 64, kvh, krow, &full[st]);
          } else {
            mbar_arrive_expect_tx(&full[st], C::V_BYTES);
#pragma unroll
            for (int x = 0; x < C::VH; ++x)
              tma_load_3d(dst + x * C::SLICE, sink ? &svmap : &vmap, x * 64, kvh, krow, &full[st]);
          }
        }
      }
      // let the copies in flight land before exit
      if (g >= 1) drain_wait(&full[(g - 1) & 1], ((g - 1) >> 1) & 1);
      if (g >= 2) drain_wait(&full[(g - 2) & 1], ((g - 2) >> 1) & 1);
      if (kq && ni >= 1) drain_wait(q_full, (ni - 1) & 1);
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(kBlk, kBlk);
      constexpr uint32_t idesc_pv = idesc_bf16_f32_bmn(kBlk, C::DV);
      // descriptors: a base per operand plus constant offsets in the 16-byte address field
      // (shared addresses stay below 256 KB, so the field never carries)
      const uint64_t qdesc0 = sw128_kmajor_desc(smem_u32(Qs));
      const uint64_t kdesc0 = sw128_kmajor_desc(smem_u32(KVs));
      const uint64_t vdesc0 = sw128_mnmajor_desc(smem_u32(KVs + C::K_BYTES), C::SLICE, 1024);
      uint32_t g = 0, ni = 0;
      bool ok = true;
      // S_g = Q K_g^T into S[g & 1].  S[g & 1] last held P_{g-2}, read by P V_{g-2}, which
      // this thread issued before: one thread's tcgen05.mma instructions execute in issue
      // order, so those reads are done before this product writes the columns -- no wait
      // for P V_{g-2} to complete, and the tensor pipe never drains between blocks.
      auto issue_qk = [&](uint32_t gg) -> bool {
        const int st = gg & 1;
        if (!mbar_wait(&k_full[st], (gg >> 1) & 1)) return false;
        tc_fence_after();
        const uint64_t kd = kdesc0 + (uint64_t)((st * C::KV_BYTES) >> 4);
#pragma unroll
        for (int kk = 0; kk < C::DQK / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::SLICE + (kk & 3) * 32;
          umma_f16_ss(tmem + (gg & 1) * C::S_COLS, qdesc0 + (uint64_t)(off >> 4),
                      kd + (uint64_t)(off >> 4), idesc_qk, kk > 0 ? 1u : 0u);
        }
        umma_commit(&s_full[gg & 1]);
        return true;
      };
      for (int kk_ = 0, i = snake_item(0, blockIdx.x, gridDim.x); ok && i < n_items;
           i = snake_item(++kk_, blockIdx.x, gridDim.x), ++ni) {
        const Item it = item_of(a, i);
        int j0, j1;
        key_range<C::BAND>(a, it, &j0, &j1);
        const int nb = key_blocks(a, it, j0, j1).n + sink_blocks<C::BAND>(a);
        if (!mbar_wait(q_full, ni & 1)) { ok = false; break; }
        if (!issue_qk(g)) { ok = false; break; }
        for (int j = 0; j < nb; ++j) {
          const uint32_t gg = g + j;
          if (j + 1 < nb && !issue_qk(gg + 1)) { ok = false; break; }
          if (j + 1 == nb) umma_commit(q_empty);  // Q free once the last S is computed
          if (!mbar_wait(&p_full[gg & 1], (gg >> 1) & 1)) { ok = false; break; }
          if (j == 0 && ni > 0 && !mbar_wait(o_empty, (ni - 1) & 1)) { ok = false; break; }
          if (!mbar_wait(&v_full[gg & 1], (gg >> 1) & 1)) { ok = false; break; }
          tc_fence_after();
          const uint64_t vd = vdesc0 + (uint64_t)(((gg & 1) * C::KV_BYTES) >> 4);
          const uint32_t p_tmem = tmem + (gg & 1) * C::S_COLS;
          const uint32_t o_tmem = tmem + C::O_COL + (C::BAND ? 0u : (gg & 1) * C::DV);
#pragma unroll
          for (int kk = 0; kk < kBlk / 16; ++kk) {
            // keys 16kk..16kk+15: 8 packed columns of P_hi at 16kk, P_lo 8 columns further;
            // V rows 16kk..: 2 swizzle atoms of 8 rows
            const uint32_t pc = 16 * kk;
            const uint64_t vdesc = vd + (uint64_t)((kk * 2048) >> 4);
            // the first block of each O (of the item's two in the selection form) overwrites it
            umma_f16_ts(o_tmem, p_tmem + pc, vdesc, idesc_pv,
                        (j >= (C::BAND ? 1 : 2) || kk > 0) ? 1u : 0u);
            umma_f16_ts(o_tmem, p_tmem + pc + 8, vdesc, idesc_pv, 1u);
          }
          umma_commit(&pv_done[gg & 1]);
        }
        g += nb;
      }
      umma_commit(mma_done);
      drain_wait(mma_done, 0);
    }
  }
  } else if (warp < kSoftWarps) {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(C::REGS_SOFT));
    if constexpr (C::BAND) {
    // ------------------------------------------------------------------ softmax, band form
    // Band items are a few key blocks long, so one group of all eight warps takes every key
    // block (no second group whose pipeline has to fill and drain every item): warp w handles
    // S columns [64 h, 64 h + 64), h = w >> 2, of the rows of TMEM quadrant w & 3 -- two
    // threads per query row, each with half of the block's keys, and one O.  The two halves
    // of a row keep one running max: each block's maxima are exchanged through shared memory
    // between the two warps of a quadrant (an mbarrier of their 64 threads per block parity,
    // waited for with the usual bound), so both take the same decisions; each keeps its own
    // part of the row sum.
    const int half = warp >> 2;
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const uint32_t t_lane = tmem + ((uint32_t)(quad * 32) << 16);
    const float ninf = __int_as_float(0xff800000);
    uint32_t g = 0, ni = 0;
    bool ok = true;
    for (int kk_ = 0, i = snake_item(0, blockIdx.x, gridDim.x); ok && i < n_items;
         i = snake_item(++kk_, blockIdx.x, gridDim.x), ++ni) {
      const Item it = item_of(a, i);
      int j0, j1;
      key_range<C::BAND>(a, it, &j0, &j1);
      const int sb = sink_blocks<C::BAND>(a);
      const KeyBlocks kb = key_blocks(a, it, j0, j1);
      const int nb = kb.n + sb;
      const int s = it.qb * kBlk + row;
      const int spos = s + a.q_off;
      const bool row_ok = s < a.S;
      float m_used = ninf, l = 0.f;
      for (int j = 0; j < nb; ++j) {
        const uint32_t gg = g + j;
        const int t0 = (j0 + j - sb) * kBlk + 64 * half;  // this half's first key
        uint32_t bits[2] = {0u, 0u};
        if (j < sb) {  // the sink block: its first nsink entries, visible to every query
#pragma unroll
          for (int w = 0; w < 2; ++w) {
            const int n = a.nsink - 64 * half - 32 * w;
            bits[w] = n >= 32 ? 0xffffffffu : (n > 0 ? (1u << n) - 1u : 0u);
          }
        } else if (row_ok) {
          // band: spos - window < t <= spos, t < T
          const int lo = max(spos - a.window + 1, 0) - t0, hi = min(spos, a.T - 1) - t0;
#pragma unroll
          for (int w = 0; w < 2; ++w) {
            const int a0 = max(lo - 32 * w, 0), a1 = min(hi - 32 * w, 31);
            bits[w] = a1 < a0 ? 0u
                              : ((a1 - a0 == 31) ? 0xffffffffu
                                                 : (((1u << (a1 - a0 + 1)) - 1u) << a0));
          }
        }
        if (!warp_wait(&s_full[gg & 1], (gg >> 1) & 1)) { ok = false; break; }
        tc_fence_after();
        const uint32_t s_col = t_lane + (gg & 1) * C::S_COLS + 64 * half;
        // This half of the row in one TMEM round trip, kept in registers; unselected keys
        // become -inf there, once.
        uint32_t r[64];
        tmem_ld32(s_col + 0, *reinterpret_cast<uint32_t(*)[32]>(r + 0));
        tmem_ld32(s_col + 32, *reinterpret_cast<uint32_t(*)[32]>(r + 32));
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (!(bits[c] & (1u << e))) r[c * 32 + e] = __float_as_uint(ninf);
        const unsigned long long scale2 = pack2(a.qk_scale, a.qk_scale);
        unsigned long long rs2 = pack2(0.f, 0.f);  // row sum, two partial sums
        // 16 keys per chunk: P = exp2(scale*s - m) (0 for unselected keys), split into bf16
        // P_hi + P_lo (P_lo = bf16(p - P_hi) keeps ~2^-17 relative precision), written over
        // the chunk's own 16 S columns; mx collects the raw maximum on the way.
        auto chunk = [&](int kk, unsigned long long nm2, float& mx) {
          uint32_t ph[8], pl[8];
#pragma unroll
          for (int e2 = 0; e2 < 8; ++e2) {
            const int e = 2 * e2;
            const float x0 = __uint_as_float(r[16 * kk + e]);
            const float x1 = __uint_as_float(r[16 * kk + e + 1]);
            mx = max3(mx, x0, x1);
            float y0, y1;
            unpack2(fma2(pack2(x0, x1), scale2, nm2), y0, y1);  // scale*s - m, two keys
            const float p0 = ex2_ftz(y0), p1 = ex2_ftz(y1);
            const unsigned long long p2 = pack2(p0, p1);
            rs2 = add2(rs2, p2);
            const __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
            const uint32_t hb = *reinterpret_cast<const uint32_t*>(&h2);
            // P_lo = bf16(p - float(P_hi)), the P_hi pair widened by bit moves
            float d0, d1;
            unpack2(sub2(p2, pack2(__uint_as_float(hb << 16), __uint_as_float(hb & 0xffff0000u))),
                    d0, d1);
            const __nv_bfloat162 l2 = __floats2bfloat162_rn(d0, d1);
            ph[e2] = hb;
            pl[e2] = *reinterpret_cast<const uint32_t*>(&l2);
          }
          tmem_st8(s_col + kk * 16, ph);
          tmem_st8(s_col + kk * 16 + 8, pl);
        };
        // One pass when every row of the warp already has a running max: P against it at once,
        // this half's block max taken on the way.  Only a row max above the running one by
        // more than 2^8 (rare after an item's first block) makes the block run again with the
        // raised max, as does a first block, whose max is taken first.  Both give the same P
        // for a row whose max stays.
        float mloc = ninf;
        const bool one_pass = __all_sync(0xffffffffu, m_used != ninf);
        if (one_pass) {
          const unsigned long long nm2 = pack2(-m_used, -m_used);
          float mx[2] = {ninf, ninf};  // two chains
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) chunk(kk, nm2, mx[kk & 1]);
          mloc = fmaxf(mx[0], mx[1]);
        } else {
          float mx[4] = {ninf, ninf, ninf, ninf};
#pragma unroll
          for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int e = 0; e < 16; e += 2)
              mx[c] = max3(mx[c], __uint_as_float(r[c * 16 + e]), __uint_as_float(r[c * 16 + e + 1]));
          mloc = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
        }
        // the row's block max: both halves' maxima, exchanged (double-buffered by block parity)
        float* xb = xch + (gg & 1) * (2 * kBlk);
        xb[half * kBlk + row] = mloc;
        uint64_t* xq = &xbar[quad * 2 + (gg & 1)];
        mbar_arrive(xq);
        if (!warp_wait(xq, (gg >> 1) & 1)) { ok = false; break; }
        const float mraw = fmaxf(mloc, xb[(half ^ 1) * kBlk + row]);
        bool again = !one_pass || __any_sync(0xffffffffu, mraw * a.qk_scale > m_used + kRescaleLog2);
        if (again && one_pass) {
          tmem_wait_st();  // the second pass writes the same columns
          rs2 = pack2(0.f, 0.f);
        }
        // a raised max rescales l now and this half of O (the item's earlier blocks) after P
        // is written, once their P V landed -- before P_j is published, so P_j V never meets
        // an unscaled O
        float alpha = 1.f;
        bool rescale_o = false, need = false;
        if (again) {
          const float mb = mraw * a.qk_scale;
          need = mb > m_used + kRescaleLog2;
          if (__any_sync(0xffffffffu, need)) {
            // whether the row has keys so far is the shared max's business, not this half's
            // sum: a half without keys yet still scales O, which the other half's keys filled
            const bool had = m_used != ninf;
            const float m_new = need ? mb : m_used;
            alpha = had ? exp2f(m_used - m_new) : 0.f;
            rescale_o = j >= 1 && __any_sync(0xffffffffu, need && had);
            if (need) {
              l *= alpha;
              m_used = m_new;
            }
          }
          const float msub = m_used == ninf ? 0.f : m_used;
          const unsigned long long nm2 = pack2(-msub, -msub);
          float mx = ninf;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) chunk(kk, nm2, mx);
        }
        {
          float r0, r1;
          unpack2(rs2, r0, r1);
          l += r0 + r1;
        }
        if (rescale_o) {
          const uint32_t gp = gg - 1;  // the previous block's P V wrote O
          if (!warp_wait(&pv_done[gp & 1], (gp >> 1) & 1)) { ok = false; break; }
          tc_fence_after();
#pragma unroll 1
          for (int c = 0; c < C::DV / 32; ++c) {
            uint32_t o[16];
            const uint32_t oc = t_lane + C::O_COL + half * (C::DV / 2) + c * 16;
            tmem_ld16(oc, o);
            tmem_wait_ld();
            if (need) {
#pragma unroll
              for (int e = 0; e < 16; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
            }
            tmem_st16(oc, o);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[gg & 1]);
      }
      if (!ok) break;
      // Band items are a few key blocks long and their output epilogue is on the path to
      // the next item's first P V: the two halves normalise and store it themselves, each
      // half of the columns (the epilogue warps stay idle).
      const uint32_t gl = g + nb - 1;  // the last block's P V completes O
      if (!warp_wait(&pv_done[gl & 1], (gl >> 1) & 1)) { ok = false; break; }
      float* mlb = ml + (ni & 1) * (2 * kBlk * 2);
      mlb[(half * kBlk + row) * 2 + 1] = l;
      mbar_arrive(&ml_full[0]);
      if (!warp_wait(&ml_full[0], ni & 1)) { ok = false; break; }
      tc_fence_after();
      const float L = mlb[(0 * kBlk + row) * 2 + 1] + mlb[(1 * kBlk + row) * 2 + 1];
      float f = L > 0.f ? 1.0f / L : 0.f;
      if (a.gate && row_ok)
        f *= gate_act(__bfloat162float(static_cast<const __nv_bfloat16*>(
                          a.gate)[((size_t)it.b * a.S + s) * a.H + it.h]),
                      a.gate_mode);
      __nv_bfloat16* orow = a.out + (((size_t)it.b * a.S + s) * a.H + it.h) * C::DV;
      // this half writes output columns [half*DV/2, (half+1)*DV/2)
#pragma unroll 1
      for (int c = 0; c < C::DV / 64; ++c) {
        const int col = half * (C::DV / 2) + c * 32;
        uint32_t r0[32];
        tmem_ld32(t_lane + C::O_COL + col, r0);
        tmem_wait_ld();
        if (row_ok) {
          uint4 v4[4];
          uint32_t* vw = reinterpret_cast<uint32_t*>(v4);
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            // a row without keys (l = 0) may hold stale values: select, never multiply
            const float y0 = L > 0.f ? __uint_as_float(r0[2 * e]) * f : 0.f;
            const float y1 = L > 0.f ? __uint_as_float(r0[2 * e + 1]) * f : 0.f;
            const __nv_bfloat162 h2 = __floats2bfloat162_rn(y0, y1);
            vw[e] = *reinterpret_cast<const uint32_t*>(&h2);
          }
          uint4* dst = reinterpret_cast<uint4*>(orow + col);
#pragma unroll
          for (int e = 0; e < 4; ++e) dst[e] = v4[e];
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(o_empty);
      g += nb;
    }
    } else {
    // ------------------------------------------------------------------ softmax
    // Group e (warps 4e..4e+3) owns the key blocks of parity e and accumulator O_e; thread =
    // query row (TMEM lane).  At the end of an item each group leaves its (m, l) in shared
    // memory for the epilogue warps and goes on with the next item.
    const int grp = warp >> 2;
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const uint32_t t_lane = tmem + ((uint32_t)(quad * 32) << 16);
    const float ninf = __int_as_float(0xff800000);
    uint32_t g = 0, ni = 0;
    bool ok = true;
    for (int kk_ = 0, i = snake_item(0, blockIdx.x, gridDim.x); ok && i < n_items;
         i = snake_item(++kk_, blockIdx.x, gridDim.x), ++ni) {
      const Item it = item_of(a, i);
      int j0, j1;
      key_range<C::BAND>(a, it, &j0, &j1);
      const int sb = sink_blocks<C::BAND>(a);
      const KeyBlocks kb = key_blocks(a, it, j0, j1);
      const int nb = kb.n + sb;
      const int s = it.qb * kBlk + row;
      const int spos = s + a.q_off;
      const bool row_ok = s < a.S;
      const uint32_t* mrow =
          (!C::BAND && row_ok) ? a.mask + ((size_t)it.b * a.S + s) * a.mask_stride : nullptr;
      const int jfirst = (int)((grp - g) & 1u);  // first block of this group's parity
      float m_used = ninf, l = 0.f;
      // the 4 selection words of key block `blk`
      auto mask_words = [&](int blk) {
        return __ldg(reinterpret_cast<const uint4*>(mrow + ((blk * kBlk) >> 5)));
      };
      // The words of this group's next block are fetched one step ahead, and the index of
      // the key block after it (from the block list) one step before that, so neither load
      // stalls the chain from S to P.
      uint4 nb4 = make_uint4(0u, 0u, 0u, 0u);
      if (mrow && jfirst < nb && jfirst >= sb) nb4 = mask_words(kb.at(jfirst - sb));
      int blk2 = (mrow && jfirst + 2 < nb) ? kb.at(jfirst + 2 - sb) : 0;
      const uint32_t o_col = C::O_COL + grp * C::DV;
      for (int j = jfirst; j < nb; j += 2) {
        const uint32_t gg = g + j;
        const int t0 = (j0 + j - sb) * kBlk;
        uint32_t bits[4] = {0u, 0u, 0u, 0u};
        if (j < sb) {  // the sink block: its first nsink entries, visible to every query
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            const int n = a.nsink - 32 * w;
            bits[w] = n >= 32 ? 0xffffffffu : (n > 0 ? (1u << n) - 1u : 0u);
          }
        } else if (!C::BAND) {
          bits[0] = nb4.x; bits[1] = nb4.y; bits[2] = nb4.z; bits[3] = nb4.w;
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
        if (!C::BAND && mrow && j + 2 < nb) {
          nb4 = mask_words(blk2);
          if (j + 4 < nb) blk2 = kb.at(j + 4 - sb);
        }
        if (!warp_wait(&s_full[gg & 1], (gg >> 1) & 1)) { ok = false; break; }
        tc_fence_after();
        const uint32_t s_col = t_lane + (gg & 1) * C::S_COLS;
        // The whole row in one TMEM round trip, kept in registers; unselected keys become
        // -inf there, once.
        uint32_t r[kBlk];
        tmem_ld32(s_col + 0, *reinterpret_cast<uint32_t(*)[32]>(r + 0));
        tmem_ld32(s_col + 32, *reinterpret_cast<uint32_t(*)[32]>(r + 32));
        tmem_ld32(s_col + 64, *reinterpret_cast<uint32_t(*)[32]>(r + 64));
        tmem_ld32(s_col + 96, *reinterpret_cast<uint32_t(*)[32]>(r + 96));
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (!(bits[c] & (1u << e))) r[c * 32 + e] = __float_as_uint(ninf);
        const unsigned long long scale2 = pack2(a.qk_scale, a.qk_scale);
        unsigned long long rs2 = pack2(0.f, 0.f);  // row sum, two partial sums
        // 16 keys per chunk: P = exp2(scale*s - m) (0 for unselected keys), split into bf16
        // P_hi + P_lo (P_lo = bf16(p - P_hi) keeps ~2^-17 relative precision), written over
        // the chunk's own 16 S columns; mx collects the raw maximum on the way.
        auto chunk = [&](int kk, unsigned long long nm2, float& mx) {
          uint32_t ph[8], pl[8];
#pragma unroll
          for (int e2 = 0; e2 < 8; ++e2) {
            const int e = 2 * e2;
            const float x0 = __uint_as_float(r[16 * kk + e]);
            const float x1 = __uint_as_float(r[16 * kk + e + 1]);
            mx = max3(mx, x0, x1);
            float y0, y1;
            unpack2(fma2(pack2(x0, x1), scale2, nm2), y0, y1);  // scale*s - m, two keys
            const float p0 = ex2_ftz(y0), p1 = ex2_ftz(y1);
            const unsigned long long p2 = pack2(p0, p1);
            rs2 = add2(rs2, p2);
            const __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
            const uint32_t hb = *reinterpret_cast<const uint32_t*>(&h2);
            // P_lo = bf16(p - float(P_hi)), the P_hi pair widened by bit moves
            float d0, d1;
            unpack2(sub2(p2, pack2(__uint_as_float(hb << 16), __uint_as_float(hb & 0xffff0000u))),
                    d0, d1);
            const __nv_bfloat162 l2 = __floats2bfloat162_rn(d0, d1);
            ph[e2] = hb;
            pl[e2] = *reinterpret_cast<const uint32_t*>(&l2);
          }
          tmem_st8(s_col + kk * 16, ph);
          tmem_st8(s_col + kk * 16 + 8, pl);
        };
        // One pass when every row of the warp already has a running max: P against it at once,
        // the block max taken on the way.  Only a block max above the running one by more than
        // 2^8 (rare after an item's first block) makes the block run again with the raised max,
        // as does a first block, whose max is taken first.  Both give the same P for a row
        // whose max stays.
        float mraw = ninf;
        bool again = true;
        if (__all_sync(0xffffffffu, m_used != ninf)) {
          const unsigned long long nm2 = pack2(-m_used, -m_used);
          float mx[2] = {ninf, ninf};  // two chains
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) chunk(kk, nm2, mx[kk & 1]);
          mraw = fmaxf(mx[0], mx[1]);
          again = __any_sync(0xffffffffu, mraw * a.qk_scale > m_used + kRescaleLog2);
          if (again) {
            tmem_wait_st();  // the second pass writes the same columns
            rs2 = pack2(0.f, 0.f);
          }
        } else {
          float mx[4] = {ninf, ninf, ninf, ninf};
#pragma unroll
          for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int e = 0; e < 32; e += 2)
              mx[c] = max3(mx[c], __uint_as_float(r[c * 32 + e]), __uint_as_float(r[c * 32 + e + 1]));
          mraw = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
        }
        // a raised max rescales l now and O_grp (this group's earlier blocks of the item) after
        // P is written, once their P V landed -- before P_j is published, so P_j V never meets
        // an unscaled O
        float alpha = 1.f;
        bool rescale_o = false, need = false;
        if (again) {
          const float mb = mraw * a.qk_scale;
          need = mb > m_used + kRescaleLog2;
          if (__any_sync(0xffffffffu, need)) {
            const float m_new = need ? mb : m_used;
            alpha = (l > 0.f) ? exp2f(m_used - m_new) : 0.f;
            rescale_o = j >= 2 && __any_sync(0xffffffffu, need && l > 0.f);
            if (need) {
              l *= alpha;
              m_used = m_new;
            }
          }
          const float msub = m_used == ninf ? 0.f : m_used;
          const unsigned long long nm2 = pack2(-msub, -msub);
          float mx = ninf;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) chunk(kk, nm2, mx);
        }
        {
          float r0, r1;
          unpack2(rs2, r0, r1);
          l += r0 + r1;
        }
        if (rescale_o) {
          if (!warp_wait(&pv_done[gg & 1], ((gg >> 1) - 1) & 1)) { ok = false; break; }
          tc_fence_after();
#pragma unroll 1
          for (int c = 0; c < C::DV / 16; ++c) {
            uint32_t o[16];
            tmem_ld16(t_lane + o_col + c * 16, o);
            tmem_wait_ld();
            if (need) {
#pragma unroll
              for (int e = 0; e < 16; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
            }
            tmem_st16(t_lane + o_col + c * 16, o);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[gg & 1]);
      }
      if (!ok) break;
      // hand this group's (m, l) to the epilogue warps; buffer ni & 1 was last read for
      // item ni - 2 (a group without blocks in an item must not run further ahead)
      const int mbuf = (int)(ni & 1);
      if (ni >= 2 && !warp_wait(&ml_empty[mbuf], ((ni >> 1) - 1) & 1)) { ok = false; break; }
      float* mlb = ml + mbuf * (2 * kBlk * 2);
      mlb[(grp * kBlk + row) * 2 + 0] = m_used;
      mlb[(grp * kBlk + row) * 2 + 1] = l;
      mbar_arrive(&ml_full[mbuf]);
      g += nb;
    }
    }
  } else {
    // every warpgroup takes part in the register split (the softmax's setmaxnreg.inc waits
    // for the registers the others give back), in band mode too, where these warps idle
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::REGS_EPI));
    if constexpr (!C::BAND) {
    // ------------------------------------------------------------------ output epilogue
    // Thread = query row (TMEM lane).  Per item: wait for the last P V of each group and for
    // the groups' (m, l); merge, normalise, gate, store bf16; free O for the next item.
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const uint32_t t_lane = tmem + ((uint32_t)(quad * 32) << 16);
    uint32_t g = 0, ni = 0;
    bool ok = true;
    for (int kk_ = 0, i = snake_item(0, blockIdx.x, gridDim.x); ok && i < n_items;
         i = snake_item(++kk_, blockIdx.x, gridDim.x), ++ni) {
      const Item it = item_of(a, i);
      int j0, j1;
      key_range<C::BAND>(a, it, &j0, &j1);
      const int nb = key_blocks(a, it, j0, j1).n + sink_blocks<C::BAND>(a);
      const int s = it.qb * kBlk + row;
      const bool row_ok = s < a.S;
      // First the groups' (m, l): a group hands them over after publishing its last P, by
      // which time the P V of its block before that has completed (its S needed the Q K^T
      // issued after that P V), so each pv_done barrier below is at most at the phase
      // waited for -- waited for earlier, a barrier one phase behind would pass on the
      // parity of the phase before.
      const int mbuf = (int)(ni & 1);
      if (!warp_wait(&ml_full[mbuf], (ni >> 1) & 1)) { ok = false; break; }
      // the last block of each parity (group): its P V completes that group's O
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int jf = (int)((e - g) & 1u);
        if (jf < nb) {
          const uint32_t gl = g + jf + ((nb - 1 - jf) & ~1);
          if (!warp_wait(&pv_done[gl & 1], (gl >> 1) & 1)) { ok = false; break; }
        }
      }
      if (!ok) break;
      tc_fence_after();
      const float* mlb = ml + mbuf * (2 * kBlk * 2);
      const float m0 = mlb[(0 * kBlk + row) * 2], l0 = mlb[(0 * kBlk + row) * 2 + 1];
      const float m1 = mlb[(1 * kBlk + row) * 2], l1 = mlb[(1 * kBlk + row) * 2 + 1];
      mbar_arrive(&ml_empty[mbuf]);
      const float M = fmaxf(m0, m1);
      const float a0 = l0 > 0.f ? exp2f(m0 - M) : 0.f;
      const float a1 = l1 > 0.f ? exp2f(m1 - M) : 0.f;
      const float L = l0 * a0 + l1 * a1;
      float f = L > 0.f ? 1.0f / L : 0.f;
      if (a.gate && row_ok)
        f *= gate_act(__bfloat162float(static_cast<const __nv_bfloat16*>(
                          a.gate)[((size_t)it.b * a.S + s) * a.H + it.h]),
                      a.gate_mode);
      const float w0 = a0 * f, w1 = a1 * f;
      __nv_bfloat16* orow = a.out + (((size_t)it.b * a.S + s) * a.H + it.h) * C::DV;
#pragma unroll 1
      for (int c = 0; c < C::DV / 16; ++c) {
        const int col = c * 16;
        uint32_t r0[16], r1[16];
        tmem_ld16(t_lane + C::O_COL + col, r0);
        tmem_ld16(t_lane + C::O_COL + C::DV + col, r1);
        tmem_wait_ld();
        if (row_ok) {
          uint4 v4[2];
          uint32_t* vw = reinterpret_cast<uint32_t*>(v4);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            // an O buffer with no weight (l = 0) may hold stale values: select, never multiply
            const float y0 = (a0 > 0.f ? __uint_as_float(r0[2 * e]) * w0 : 0.f) +
                             (a1 > 0.f ? __uint_as_float(r1[2 * e]) * w1 : 0.f);
            const float y1 = (a0 > 0.f ? __uint_as_float(r0[2 * e + 1]) * w0 : 0.f) +
                             (a1 > 0.f ? __uint_as_float(r1[2 * e + 1]) * w1 : 0.f);
            const __nv_bfloat162 h2 = __floats2bfloat162_rn(y0, y1);
            vw[e] = *reinterpret_cast<const uint32_t*>(&h2);
          }
          uint4* dst = reinterpret_cast<uint4*>(orow + col);
          dst[0] = v4[0];
          dst[1] = v4[1];
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(o_empty);
      g += nb;
    }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// The block list of a selection mask, per (batch row, 128-query block): the key blocks of 128
// that hold a selected key of any of its queries, in ascending order, in list[0 .. count).  A
// query block that selected nothing gets the one block 0 (every key of it masked).
__global__ void __launch_bounds__(256) block_list_kernel(const uint32_t* __restrict__ mask,
                                                         int mask_stride, int S, int T, int q_off,
                                                         int nqb, int nkb,
                                                         int* __restrict__ count,
                                                         uint16_t* __restrict__ list) {
  // One CTA per (b, query block).  G threads share a key block, each over every G-th row,
  // eight independent row loads at a time; a thread stops at the first selected key, or once
  // another thread has marked the block.  Key blocks past the query block's last causal key
  // hold no selection and are not read.
  extern __shared__ uint32_t occ[];
  const int b = blockIdx.x / nqb, qb = blockIdx.x % nqb;
  const int s0 = qb * kBlk, rows = min(S, s0 + kBlk) - s0;
  const int t_hi = min(T - 1, s0 + rows - 1 + q_off);
  const int jn = t_hi < 0 ? 0 : min(nkb, t_hi / kBlk + 1);
  const int nw = (jn + 31) >> 5;
  const uint32_t* m0 = mask + ((size_t)b * S + s0) * mask_stride;
  uint16_t* out = list + (size_t)blockIdx.x * nkb;
  for (int i = threadIdx.x; i < nw; i += blockDim.x) occ[i] = 0u;
  __syncthreads();
  int G = 1;
  while (G < 16 && 2 * G * jn <= (int)blockDim.x) G *= 2;
  for (int i = threadIdx.x; i < jn * G; i += blockDim.x) {
    const int j = i % jn, g = i / jn;
    const uint4* col = reinterpret_cast<const uint4*>(m0) + j;
    bool any = false;
    for (int r0 = g; r0 < rows && !any; r0 += 8 * G) {
      uint32_t o = 0u;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int s = r0 + k * G;
        if (s < rows) {
          const uint4 v = __ldg(col + (size_t)s * (mask_stride >> 2));
          o |= v.x | v.y | v.z | v.w;
        }
      }
      any = o != 0u;
      if (!any && ((*(volatile uint32_t*)&occ[j >> 5] >> (j & 31)) & 1u)) break;
    }
    if (any) atomicOr(&occ[j >> 5], 1u << (j & 31));
  }
  __syncthreads();
  if (threadIdx.x < 32) {  // warp 0 compacts the marked blocks in ascending order
    const int lane = threadIdx.x;
    int base = 0;
    for (int w0 = 0; w0 < nw; w0 += 32) {
      const int w = w0 + lane;
      uint32_t bits = w < nw ? occ[w] : 0u;
      const int c = __popc(bits);
      int incl = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      int pos = base + incl - c;
      while (bits) {
        out[pos++] = (uint16_t)(w * 32 + __ffs(bits) - 1);
        bits &= bits - 1u;
      }
      base += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) {
      if (base == 0) {  // nothing selected: one block, every key of it masked
        out[0] = 0;
        base = 1;
      }
      count[blockIdx.x] = base;
    }
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
                      const int* bcount, const uint16_t* blist, cudaStream_t st) {
  CUtensorMap qm, km, vm, skm, svm;
  if (!map3d(&qm, p.q, (uint64_t)p.B * p.S, p.H, C::DQK) ||
      !map3d(&km, p.k, (uint64_t)p.B * p.T, p.HKV, C::DQK) ||
      !map3d(&vm, p.v, (uint64_t)p.B * p.T, p.HKV, C::DV))
    return cudaErrorInvalidValue;
  const bool sinks = p.sink_k != nullptr && p.nsink > 0;
  if (sinks) {
    if (p.nsink > kBlk) return cudaErrorNotSupported;  // one sink block per item
    if (!map3d(&skm, p.sink_k, (uint64_t)p.nsink, p.HKV, C::DQK) ||
        !map3d(&svm, p.sink_v, (uint64_t)p.nsink, p.HKV, C::DV))
      return cudaErrorInvalidValue;
  } else {
    skm = km;  // unused
    svm = vm;
  }
  AttnArgs a{};
  a.mask = mask; a.gate = p.gate; a.out = static_cast<__nv_bfloat16*>(p.out);
  a.gate_mode = p.gate_mode; a.qk_scale = p.sm_scale * kLog2e;
  a.B = p.B; a.S = p.S; a.T = p.T; a.H = p.H; a.HKV = p.HKV; a.q_off = p.q_off;
  a.window = p.window; a.mask_stride = mask_stride;
  a.nsink = sinks ? p.nsink : 0;
  a.nqb = (p.S + kBlk - 1) / kBlk;
  a.bcount = bcount;
  a.blist = blist;
  a.nkb = (p.T + kBlk - 1) / kBlk;
  const int items = p.B * p.H * a.nqb;
  const int nsm = num_sms();
  // the K/V all items read; above the L2 size (126 MB on B200) the bands (half as many
  // query blocks as SMs) keep about two heads' K/V in use at a time
  const double kv_bytes = (double)p.B * p.T * p.HKV * (C::DQK + C::DV) * 2.0;
  a.band = kv_bytes > 96.0 * (1 << 20) ? (nsm / 2 > 1 ? nsm / 2 : 1) : 0;
  const int grid = items < nsm ? items : nsm;
  auto kern = masked_attn_tc_kernel<C>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  // the register split only completes if the launch holds the registers it hands out
  static const int launch_regs = [&] {
    cudaFuncAttributes fa{};
    return cudaFuncGetAttributes(&fa, kern) == cudaSuccess ? fa.numRegs : 0;
  }();
  if (launch_regs * C::THREADS < 2 * 128 * C::REGS_SOFT + 128 * C::REGS_CTL + 128 * C::REGS_EPI)
    return cudaErrorInvalidConfiguration;
  kern<<<grid, C::THREADS, C::SMEM, st>>>(qm, km, vm, skm, svm, a);
  return cudaGetLastError();
}

}  // namespace

bool masked_attn_supported(int dtype, int DQK, int DV) {
  return dtype == 1 && (DQK == 128 || DQK == 192) && DV == 128;
}

cudaError_t launch_masked_attn(const AttnProblem& p, const uint32_t* mask, int mask_stride,
                               void* blocks, cudaStream_t st) {
  if (!masked_attn_supported(p.dtype, p.DQK, p.DV)) return cudaErrorNotSupported;
  const bool band = p.idx == nullptr && mask == nullptr;
  if (!band && mask == nullptr) return cudaErrorInvalidValue;
  const int* bcount = nullptr;
  const uint16_t* blist = nullptr;
  if (!band && blocks != nullptr) {  // the key blocks each 128-query block selected from
    const int nqb = (p.S + kBlk - 1) / kBlk;
    const int nkb = (p.T + kBlk - 1) / kBlk;
    int* cnt = static_cast<int*>(blocks);
    uint16_t* lst = reinterpret_cast<uint16_t*>(cnt + (size_t)p.B * nqb);
    const size_t occ_bytes = (size_t)((nkb + 31) / 32) * sizeof(uint32_t);
    block_list_kernel<<<(unsigned)(p.B * nqb), 256, occ_bytes, st>>>(
        mask, mask_stride, p.S, p.T, p.q_off, nqb, nkb, cnt, lst);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    bcount = cnt;
    blist = lst;
  }
  if (p.DQK == 128)
    return band ? launch_fa<FaCfg<128, 128, true>>(p, mask, mask_stride, bcount, blist, st)
                : launch_fa<FaCfg<128, 128, false>>(p, mask, mask_stride, bcount, blist, st);
  return band ? launch_fa<FaCfg<192, 128, true>>(p, mask, mask_stride, bcount, blist, st)
              : launch_fa<FaCfg<192, 128, false>>(p, mask, mask_stride, bcount, blist, st);
}

}  // namespace dsa
