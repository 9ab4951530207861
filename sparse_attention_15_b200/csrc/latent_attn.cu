// Sparse attention over a shared latent cache (the MQA form of MLA) on tcgen05.
//
// [AXK2] "注意力前向的骨架：MLA + 显式稀疏掩码", step 2: kv_a_proj_with_mqa compresses keys and
// values into one latent vector per token (kv_lora_rank dims) plus a RoPE key slice shared
// by all heads; [AXK2] "注意力后端选择": the indexer's positions (indices=sparse_indices) are
// meant for flash-mla (flash_mla_with_kvcache), which attends over that latent cache.  With
// the key and value up-projections absorbed into the query and the output, every head
// attends over the same cached row c[t] = [latent | rope] (DQK = 512 + 64 = 576 dims): the
// logit of head h is sm_scale * q[h,:] . c[t,:] and its output is sum_t p[h,t] c[t, 0:DV]
// (DV = 512, the latent part).  [PANGU] §3.4: for MLA the PAS sinks are latent KV rows,
// visible to every query.
//
// Because the key row is shared by all heads, a block of selected keys is a real
// [H x DQK] . [DQK x keys] tensor-core product: S = Q C^T with M = 128 heads (rows past H
// are zero), N = 48 keys, K = 576; then O += P V with M = 128 heads, N = 256, K = 48 keys.
// O for all 512 latent columns would fill the whole tensor memory, so every (query row, key
// split) is computed by two CTAs, one per half of DV; each computes the full S (the QK
// product is repeated, nothing is exchanged between CTAs) and the two run side by side, so
// the second reads the gathered rows from L2.  A block is 36 QK and 6 PV instructions: the
// MMA issue rate, not the tensor pipe, bounds this kernel, so the blocks are as wide as the
// memory budgets allow while three of them stay in flight.
//
// Tensor memory (512 columns): Q dims 0..319 as the tensor-memory A operand of QK (5 x 32
// columns of bf16 pairs, so those MMAs read only the key tile from shared memory), S0, S1
// (48 columns each; P_hi / P_lo are written over them), O (256 columns).  Shared memory:
// Q dims 320..575 (4 K-major slices with the 128-byte swizzle) and a ring of 3 key blocks
// (48 rows x 576 dims, 9 slices).  The same bytes of a key block are the K-major B operand
// of QK and, for the DV/2 columns of this CTA, the MN-major B operand of PV.  P is split into
// bf16 P_hi + P_lo (as in the masked-tile kernel) to keep float32 probability precision.
//
// Roles: warps 0..3 softmax and epilogue (thread = head = TMEM lane; they also write Q's
// tensor-memory part), warp 4 MMA issuer and TMEM owner, warps 5..8 gather the selected rows
// with 16-byte cp.async into the swizzled ring (zero fill for skipped entries), 12 rows of
// every block each.  Every wait is bounded.
#include <climits>

#include "common.cuh"
#include "kernels.h"

namespace dsa {

namespace {

constexpr int kDQK = 576, kDV = 512, kNV = kDV / 2;  // N of PV per CTA
constexpr int kNK = 48;                              // keys per block (N of QK)
constexpr int kSlices = kDQK / 64;                   // 64-dim slices of a row
constexpr int kQT = 5;                               // Q slices in tensor memory
constexpr int kQS = kSlices - kQT;                   // Q slices in shared memory
constexpr int kStages = 3;                           // key blocks in the ring
constexpr int kSB = 2;                               // S buffers
constexpr int kKSlice = kNK * 128;                   // one slice of a key block (bytes)
constexpr int kStageBytes = kSlices * kKSlice;
constexpr int kQSlice = 128 * 128;                   // one slice of Q (128 rows)
constexpr int kQBytes = kQS * kQSlice;
constexpr int kBarBytes = 256;
// no alignment slack: the dynamic shared memory of a kernel without static shared memory
// starts 1024-byte aligned (checked at run time)
constexpr int kSmem = kQBytes + kStages * kStageBytes + kBarBytes;
constexpr uint32_t kColQ = 0, kColS = kQT * 32, kColO = kColS + kSB * kNK;
constexpr int kWarpMma = 4, kWarpProd0 = 5, kProdThreads = 128;
constexpr int kThreads = 32 * 9;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleLog2 = 8.0f;
static_assert(kColO + kNV == 512, "TMEM budget");
static_assert(kSmem <= 227 * 1024, "shared memory budget");
constexpr int kKeysPerWarp = kNK / 4;                // producer warp share of a block
static_assert(kNK % 16 == 0 && kKeysPerWarp <= 32, "block split");
static_assert(kKSlice % 1024 == 0, "swizzle atoms");

struct LatentArgs {
  const __nv_bfloat16* q;     // [rows, H, 576]
  const __nv_bfloat16* kv;    // [B, T, 576]
  const int32_t* idx;         // [rows, K]
  const __nv_bfloat16* sink;  // [nsink, 576] or NULL
  const __nv_bfloat16* gate;  // [rows, H] or NULL
  __nv_bfloat16* out;         // [rows, H, 512]
  float* part_o;              // [rows, nsplit, H, 512] (split mode)
  float* part_ml;             // [rows, nsplit, H, 2]
  float qk_scale;             // sm_scale * log2(e)
  int S, T, H, K, q_off, nsink, gate_mode;
  int nsplit, kps;            // key splits per row, entries per split (multiple of kNK)
};

__device__ __forceinline__ void cp_async16(void* dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src),
               "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Source row of entry p of a query's key list -- the nsink sinks first, then the selected
// positions -- or NULL when the entry is skipped (past the split, -1, out of range, future).
__device__ __forceinline__ const __nv_bfloat16* key_row(const LatentArgs& a,
                                                        const int32_t* idx_row, int b,
                                                        int spos, int p, int p1) {
  if (p >= p1) return nullptr;
  if (p < a.nsink) return a.sink + (size_t)p * kDQK;
  const int t = __ldg(idx_row + (p - a.nsink));
  if (t < 0 || t >= a.T || t > spos) return nullptr;
  return a.kv + ((size_t)b * a.T + t) * kDQK;
}

__global__ void __launch_bounds__(kThreads, 1) latent_attn_kernel(const LatentArgs a) {
  extern __shared__ __align__(1024) uint8_t smem[];
  if ((smem_u32(smem) & 1023u) != 0u) {  // the swizzled layout needs 1024-byte atoms
    if (threadIdx.x == 0) flag_status(kStatusInternal);
    return;
  }
  uint8_t* Qs = smem;                 // [kQS] slices of [128 rows x 64]
  uint8_t* ring = smem + kQBytes;     // [kStages] key blocks
  uint64_t* bars = reinterpret_cast<uint64_t*>(ring + kStages * kStageBytes);
  uint64_t* full = bars;              // [3] key block landed (producer threads)
  uint64_t* empty = bars + 3;         // [3] key block consumed by its P V
  uint64_t* s_full = bars + 6;        // [2] S = Q C^T done
  uint64_t* p_full = bars + 8;        // [2] P written (softmax warps)
  uint64_t* pv_done = bars + 10;      // [2] O += P V of that block done
  uint64_t* q_full = bars + 12;       // Q shared-memory part landed (producer threads)
  uint64_t* q_tm = bars + 13;         // Q tensor-memory part written (softmax warps)
  uint64_t* mma_done = bars + 14;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 15);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // item = (query row, key split, DV half); the two halves of a split are neighbours
  const int hv = blockIdx.x & 1;
  const int rs = blockIdx.x >> 1;
  const int sp = rs % a.nsplit;
  const int r = rs / a.nsplit;
  const int b = r / a.S;
  const int spos = r % a.S + a.q_off;
  const int nkeys = a.nsink + a.K;
  const int p0 = sp * a.kps;
  const int p1 = min(nkeys, p0 + a.kps);
  const int NB = (p1 - p0 + kNK - 1) / kNK;
  const int32_t* idx_row = a.idx + (size_t)r * a.K;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full[i], kProdThreads);  // every producer thread copies part of a block
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < kSB; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 4);
      mbar_init(&pv_done[i], 1);
    }
    mbar_init(q_full, kProdThreads);
    mbar_init(q_tm, 4);
    mbar_init(mma_done, 1);
    fence_mbar_init();
  }
  if (warp == kWarpMma) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp >= kWarpProd0) {
    // ------------------------------------------------------------------ gather producers
    const int p = threadIdx.x - kWarpProd0 * 32;
    bool ok = true;
    // Q dims 320..575 of every head: 128 rows x 32 chunks of 16 bytes
    {
      const __nv_bfloat16* q0 = a.q + (size_t)r * a.H * kDQK;
#pragma unroll 4
      for (int i = 0; i < kQS * 8; ++i) {
        const int e = p + kProdThreads * i;
        const int row = e / (kQS * 8), k = e - row * (kQS * 8);
        const int x = k >> 3, cc = k & 7;
        const bool in = row < a.H;
        const __nv_bfloat16* src = in ? q0 + (size_t)row * kDQK + (kQT + x) * 64 + cc * 8 : a.q;
        cp_async16(Qs + x * kQSlice + row * 128 + ((cc ^ (row & 7)) << 4), src, in ? 16u : 0u);
      }
      cp_async_commit();
    }
    // All four producer warps copy every block, warp w its 12 keys 12w..12w+11: each waits
    // for its own copies, fences and arrives, so a block is published as soon as its last
    // rows land.  Lane l < 12 resolves entry 12w + l of the block (read one block ahead) and
    // copies chunks l, l+32, l+64 (< 72) of every row: chunk c is slice c/8, 16-byte column
    // c%8, swizzled by the row's index mod 8.
    const int lane_p = p & 31;
    const int kq = (p >> 5) * kKeysPerWarp;  // first key of this warp in a block
    const int le = lane_p < kKeysPerWarp ? lane_p : 0;  // the entry this lane resolves
    const __nv_bfloat16* nxt = NB > 0 ? key_row(a, idx_row, b, spos, p0 + kq + le, p1) : nullptr;
    uint32_t dst_off[3], src_off[3], cc_of[3];
#pragma unroll
    for (int m = 0; m < 3; ++m) {
      const int c = lane_p + 32 * m;
      cc_of[m] = c & 7;
      dst_off[m] = (c >> 3) * kKSlice;
      src_off[m] = (c >> 3) * 64 + (c & 7) * 8;
    }
    bool q_pending = true;  // this thread's Q copies not yet published
    for (int j = 0; j < NB; ++j) {
      const int st = j % kStages;
      const unsigned long long cur = reinterpret_cast<unsigned long long>(nxt);
      if (j + 1 < NB) nxt = key_row(a, idx_row, b, spos, p0 + (j + 1) * kNK + kq + le, p1);
      // warp-uniform wait: the whole warp takes part in the shuffles below
      if (j >= kStages && !warp_wait(&empty[st], ((j / kStages) - 1) & 1)) { ok = false; break; }
      uint8_t* stage = ring + st * kStageBytes;
#pragma unroll 4
      for (int i = 0; i < kKeysPerWarp; ++i) {
        const __nv_bfloat16* row =
            reinterpret_cast<const __nv_bfloat16*>(__shfl_sync(0xffffffffu, cur, i));
        const int key = kq + i;  // row of the block; its 128-byte lines swizzle by key % 8
#pragma unroll
        for (int m = 0; m < 3; ++m) {
          if (m == 2 && lane_p >= kDQK / 8 - 64) break;
          cp_async16(stage + dst_off[m] + key * 128 + ((cc_of[m] ^ (key & 7)) << 4),
                     row ? row + src_off[m] : a.kv, row ? 16u : 0u);
        }
      }
      cp_async_commit();
      if (q_pending) {  // the Q group (committed first) has landed
        cp_async_wait<1>();
        fence_proxy_async_smem();
        mbar_arrive(q_full);
        q_pending = false;
      }
      cp_async_wait<0>();
      fence_proxy_async_smem();
      mbar_arrive(&full[st]);
    }
    cp_async_wait<0>();
    if (ok && q_pending) {  // no blocks: still publish the Q copies
      fence_proxy_async_smem();
      mbar_arrive(q_full);
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, kNK);
      constexpr uint32_t idesc_pv = idesc_bf16_f32_bmn(128, kNV);
      bool ok = mbar_wait(q_full, 0) && mbar_wait(q_tm, 0);
      // descriptors: a base per operand plus constant offsets in the 16-byte address field
      // (shared addresses stay below 256 KB, so the field never carries)
      const uint64_t qdesc0 = sw128_kmajor_desc(smem_u32(Qs));
      const uint64_t kdesc0 = sw128_kmajor_desc(smem_u32(ring));
      // S_j = Q C_j^T into S[j % 2] (the buffer last held P_{j-2}); O += P_j V_j.  Issued in
      // whatever order their inputs arrive: a P V never waits behind the next block's load.
      auto issue_qk = [&](int j) {
        const int st = j % kStages, sb = j % kSB;
        const uint64_t kd = kdesc0 + (uint64_t)(st * (kStageBytes >> 4));
        const uint32_t d = tmem + kColS + sb * kNK;
#pragma unroll
        for (int x = 0; x < kSlices; ++x)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t bdesc = kd + (uint64_t)((x * kKSlice + kk * 32) >> 4);
            const uint32_t acc = (x | kk) ? 1u : 0u;
            if (x < kQT)
              umma_f16_ts(d, tmem + kColQ + x * 32 + kk * 8, bdesc, idesc_qk, acc);
            else
              umma_f16_ss(d, qdesc0 + (uint64_t)(((x - kQT) * kQSlice + kk * 32) >> 4), bdesc,
                          idesc_qk, acc);
          }
        umma_commit(&s_full[sb]);
      };
      auto issue_pv = [&](int j) {
        const int sb = j % kSB, st = j % kStages;
        // V = the first DV columns of the key rows; this CTA's half starts at slice 4*hv
        const uint64_t vd = sw128_mnmajor_desc(smem_u32(ring + st * kStageBytes) +
                                              (uint32_t)(4 * hv * kKSlice), kKSlice, 1024);
        const uint32_t pt = tmem + kColS + sb * kNK;
#pragma unroll
        for (int c = 0; c < kNK / 16; ++c) {
          // keys 16c..16c+15: P_hi in 8 columns at 16c, P_lo 8 further; 2 atoms of V rows
          const uint64_t vdesc = vd + (uint64_t)((c * 2048) >> 4);
          umma_f16_ts(tmem + kColO, pt + 16 * c, vdesc, idesc_pv, (j > 0 || c > 0) ? 1u : 0u);
          umma_f16_ts(tmem + kColO, pt + 16 * c + 8, vdesc, idesc_pv, 1u);
        }
        umma_commit(&empty[st]);
        umma_commit(&pv_done[sb]);
      };
      // nq: next S to compute, np: next P V.  S_nq needs its key block and, for nq >= 2, the
      // P V of block nq-2 (issued: np >= nq-1) to have finished with the buffer.  Every
      // phase tested here is the one after the last phase consumed, so a parity test is
      // unambiguous.  No progress for the wait limit -> timeout.
      int nq = 0, np = 0;
      long long t_prog = clock64();
      while (ok && np < NB) {
        bool prog = false;
        if (nq < NB && (nq < kSB || np >= nq - 1) &&
            mbar_try_wait(&full[nq % kStages], (nq / kStages) & 1) &&
            (nq < kSB || mbar_try_wait(&pv_done[nq % kSB], ((nq / kSB) - 1) & 1))) {
          tc_fence_after();
          issue_qk(nq++);
          prog = true;
        }
        if (np < nq && mbar_try_wait(&p_full[np % kSB], (np / kSB) & 1)) {
          tc_fence_after();
          issue_pv(np++);
          prog = true;
        }
        if (prog) {
          t_prog = clock64();
        } else if (timeout_recorded() || clock64() - t_prog > kWaitCycles) {
          flag_status(kStatusTimeout);
          ok = false;
        }
      }
      umma_commit(mma_done);
      drain_wait(mma_done, 0);
    }
  } else {
    // ------------------------------------------------------------------ softmax + epilogue
    const int h = warp * 32 + lane;
    const bool head_ok = h < a.H;
    const uint32_t t_lane = tmem + ((uint32_t)(warp * 32) << 16);
    const float ninf = __int_as_float(0xff800000);
    bool ok = true;
    // Q dims 0..319 of head h -> TMEM columns kColQ.. (bf16 pairs; zeros for h >= H), in
    // batches of two slices, each batch's loads all in flight before its stores
    {
      const uint4* src = reinterpret_cast<const uint4*>(a.q + ((size_t)r * a.H + h) * kDQK);
#pragma unroll
      for (int x0 = 0; x0 < kQT; x0 += 2) {
        uint4 u[16];
#pragma unroll
        for (int c = 0; c < 16; ++c)
          u[c] = (head_ok && x0 * 8 + c < kQT * 8) ? __ldg(src + x0 * 8 + c)
                                                   : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int x = 0; x < 2; ++x) {
          if (x0 + x >= kQT) break;
          uint32_t v[32];
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            v[4 * c] = u[x * 8 + c].x; v[4 * c + 1] = u[x * 8 + c].y;
            v[4 * c + 2] = u[x * 8 + c].z; v[4 * c + 3] = u[x * 8 + c].w;
          }
          tmem_st32(t_lane + kColQ + (x0 + x) * 32, v);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(q_tm);
    }
    float m_used = ninf, l = 0.f;
    for (int j = 0; j < NB; ++j) {
      const int sb = j % kSB;
      // which of the block's 48 entries are attended (the same for every head)
      const int e0 = p0 + j * kNK + lane;
      const uint32_t bits0 =
          __ballot_sync(0xffffffffu, key_row(a, idx_row, b, spos, e0, p1) != nullptr);
      const uint32_t bits1 = __ballot_sync(
          0xffffffffu, lane < kNK - 32 && key_row(a, idx_row, b, spos, e0 + 32, p1) != nullptr);
      if (!warp_wait(&s_full[sb], (j / kSB) & 1)) { ok = false; break; }
      tc_fence_after();
      const uint32_t s_col = t_lane + kColS + sb * kNK;
      uint32_t rr[48];
      tmem_ld32(s_col, *reinterpret_cast<uint32_t(*)[32]>(rr));
      tmem_ld16(s_col + 32, *reinterpret_cast<uint32_t(*)[16]>(rr + 32));
      tmem_wait_ld();
      float mx0 = ninf, mx1 = ninf;
#pragma unroll
      for (int e = 0; e < 32; e += 2) {
        mx0 = fmaxf(mx0, (bits0 >> e) & 1u ? __uint_as_float(rr[e]) : ninf);
        mx1 = fmaxf(mx1, (bits0 >> (e + 1)) & 1u ? __uint_as_float(rr[e + 1]) : ninf);
      }
#pragma unroll
      for (int e = 0; e < 16; e += 2) {
        mx0 = fmaxf(mx0, (bits1 >> e) & 1u ? __uint_as_float(rr[32 + e]) : ninf);
        mx1 = fmaxf(mx1, (bits1 >> (e + 1)) & 1u ? __uint_as_float(rr[33 + e]) : ninf);
      }
      const float mb = fmaxf(mx0, mx1) * a.qk_scale;
      // the running max is raised (and O, l rescaled) only when a block max exceeds it by
      // more than 2^8, so exp2 arguments stay <= 8 and rescales are rare
      const bool need = mb > m_used + kRescaleLog2;
      if (__any_sync(0xffffffffu, need)) {
        const float m_new = need ? mb : m_used;
        const float alpha = (l > 0.f) ? exp2f(m_used - m_new) : 0.f;
        if (j >= 1 && __any_sync(0xffffffffu, need && l > 0.f)) {
          // O holds blocks 0..j-1: rescale once the last of their P V products landed
          const int jp = j - 1;
          if (!warp_wait(&pv_done[jp % kSB], (jp / kSB) & 1)) { ok = false; break; }
          tc_fence_after();
#pragma unroll 1
          for (int c = 0; c < kNV / 16; ++c) {
            uint32_t o[16];
            tmem_ld16(t_lane + kColO + c * 16, o);
            tmem_wait_ld();
            if (need) {
#pragma unroll
              for (int e = 0; e < 16; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
            }
            tmem_st16(t_lane + kColO + c * 16, o);
          }
          tmem_wait_st();
        }
        if (need) {
          l *= alpha;
          m_used = m_new;
        }
      }
      // P = exp2(scale*s - m) for attended entries, 0 otherwise, as bf16 P_hi + P_lo written
      // over the chunk's own 16 S columns
      const float msub = m_used == ninf ? 0.f : m_used;
      float rs0 = 0.f, rs1 = 0.f;
#pragma unroll
      for (int c = 0; c < kNK / 16; ++c) {
        const uint32_t bw = (c < 2 ? bits0 : bits1) >> (16 * (c & 1));
        uint32_t ph[8], pl[8];
#pragma unroll
        for (int e2 = 0; e2 < 8; ++e2) {
          const int e = 2 * e2;
          const float x0 = (bw >> e) & 1u ? __uint_as_float(rr[16 * c + e]) : ninf;
          const float x1 = (bw >> (e + 1)) & 1u ? __uint_as_float(rr[16 * c + e + 1]) : ninf;
          const float y0 = ex2_ftz(fmaf(x0, a.qk_scale, -msub));
          const float y1 = ex2_ftz(fmaf(x1, a.qk_scale, -msub));
          rs0 += y0;
          rs1 += y1;
          const __nv_bfloat162 h2 = __floats2bfloat162_rn(y0, y1);
          const uint32_t hb = *reinterpret_cast<const uint32_t*>(&h2);
          const __nv_bfloat162 l2 = __floats2bfloat162_rn(y0 - __uint_as_float(hb << 16),
                                                          y1 - __uint_as_float(hb & 0xffff0000u));
          ph[e2] = hb;
          pl[e2] = *reinterpret_cast<const uint32_t*>(&l2);
        }
        tmem_st8(s_col + 16 * c, ph);
        tmem_st8(s_col + 16 * c + 8, pl);
      }
      l += rs0 + rs1;
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[sb]);
    }
    // ---------------- epilogue: normalise (or keep the split's partial), gate, store
    if (ok && NB > 0) {
      const int jl = NB - 1;
      ok = warp_wait(&pv_done[jl % kSB], (jl / kSB) & 1);
    }
    if (ok) {
      tc_fence_after();
      if (a.nsplit == 1) {
        float f = l > 0.f ? 1.0f / l : 0.f;
        if (a.gate && head_ok)
          f *= gate_act(__bfloat162float(a.gate[(size_t)r * a.H + h]), a.gate_mode);
        __nv_bfloat16* orow = a.out + ((size_t)r * a.H + h) * kDV + hv * kNV;
#pragma unroll 1
        for (int c = 0; c < kNV / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(t_lane + kColO + c * 32, o);
          tmem_wait_ld();
          if (head_ok) {
            uint4 v4[4];
            uint32_t* vw = reinterpret_cast<uint32_t*>(v4);
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const __nv_bfloat162 h2 = __floats2bfloat162_rn(__uint_as_float(o[2 * e]) * f,
                                                              __uint_as_float(o[2 * e + 1]) * f);
              vw[e] = *reinterpret_cast<const uint32_t*>(&h2);
            }
            uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
            for (int e = 0; e < 4; ++e) dst[e] = v4[e];
          }
        }
      } else {
        const size_t pi = ((size_t)r * a.nsplit + sp) * a.H + h;
        float* po = a.part_o + pi * kDV + hv * kNV;
#pragma unroll 1
        for (int c = 0; c < kNV / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(t_lane + kColO + c * 32, o);
          tmem_wait_ld();
          if (head_ok) {
            float4* dst = reinterpret_cast<float4*>(po + c * 32);
#pragma unroll
            for (int e = 0; e < 8; ++e)
              dst[e] = make_float4(__uint_as_float(o[4 * e]), __uint_as_float(o[4 * e + 1]),
                                   __uint_as_float(o[4 * e + 2]), __uint_as_float(o[4 * e + 3]));
          }
        }
        // both halves hold the same (m, l): the first writes them
        if (hv == 0 && head_ok) {
          a.part_ml[pi * 2] = l > 0.f ? m_used : ninf;
          a.part_ml[pi * 2 + 1] = l;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Key splits per query row: the count whose waves of CTA pairs (one CTA per SM, 148 SMs)
// finish first, counting each item's set-up (the Q load) as about two key blocks.  A fixed
// SM count keeps the workspace size a function of the shape alone.
void latent_split(int rows, int nkeys, int* nsplit, int* kps) {
  const int blocks = (nkeys + kNK - 1) / kNK;
  long long best_cost = LLONG_MAX;
  int best_n = 1, best_bps = blocks;
  for (int ns = 1; ns <= 64 && ns <= blocks; ++ns) {
    const int bps = (blocks + ns - 1) / ns;
    const int n = (blocks + bps - 1) / bps;
    const long long items = 2LL * rows * n;
    const long long waves = (items + 147) / 148;
    const long long cost = waves * (bps + 2);
    if (cost < best_cost) {
      best_cost = cost;
      best_n = n;
      best_bps = bps;
    }
  }
  *nsplit = best_n;
  *kps = best_bps * kNK;
}

}  // namespace

bool latent_attn_supported(int dtype, int H, int DQK, int DV) {
  return dtype == 1 && DQK == kDQK && DV == kDV && H >= 1 && H <= 128;
}

size_t latent_attn_workspace_bytes(int B, int S, int H, int K, int nsink) {
  const long long rows = (long long)B * S;
  if (rows <= 0 || K + nsink <= 0) return 0;
  int ns, kps;
  latent_split((int)rows, K + nsink, &ns, &kps);
  if (ns == 1) return 0;
  return (size_t)rows * ns * H * (kDV + 2) * sizeof(float);
}

cudaError_t launch_latent_attn(const LatentProblem& p, void* ws, size_t ws_bytes,
                               cudaStream_t st) {
  if (!latent_attn_supported(p.dtype, p.H, p.DQK, p.DV)) return cudaErrorNotSupported;
  const long long rows = (long long)p.B * p.S;
  if (rows == 0) return cudaSuccess;
  LatentArgs a{};
  a.q = static_cast<const __nv_bfloat16*>(p.q);
  a.kv = static_cast<const __nv_bfloat16*>(p.kv);
  a.idx = p.idx;
  a.sink = static_cast<const __nv_bfloat16*>(p.sink);
  a.nsink = p.sink ? p.nsink : 0;
  a.gate = static_cast<const __nv_bfloat16*>(p.gate);
  a.gate_mode = p.gate_mode;
  a.out = static_cast<__nv_bfloat16*>(p.out);
  a.qk_scale = p.sm_scale * kLog2e;
  a.S = p.S; a.T = p.T; a.H = p.H; a.K = p.K; a.q_off = p.q_off;
  latent_split((int)rows, a.nsink + a.K, &a.nsplit, &a.kps);
  if (a.nsplit > 1) {
    const size_t need = (size_t)rows * a.nsplit * p.H * (kDV + 2) * sizeof(float);
    if (ws == nullptr || ws_bytes < need) return cudaErrorInvalidValue;
    a.part_o = static_cast<float*>(ws);
    a.part_ml = a.part_o + (size_t)rows * a.nsplit * p.H * kDV;
  }
  const long long grid = rows * a.nsplit * 2;
  if (grid > 0x7fffffffLL) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(latent_attn_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
  if (e != cudaSuccess) return e;
  latent_attn_kernel<<<(unsigned)grid, kThreads, kSmem, st>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess || a.nsplit == 1) return e;
  return launch_split_combine(1, a.part_o, a.part_ml, (int)rows, a.nsplit, p.H, kDV, p.gate,
                              p.gate_mode, p.out, st);
}

}  // namespace dsa
