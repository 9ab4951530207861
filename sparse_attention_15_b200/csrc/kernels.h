// Host-side launchers of the libdsa kernels (internal; the public ABI is include/dsa.h).
// Every launcher only enqueues work and returns the launch error, if any.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace dsa {

// Sets the thread-local text returned by dsa_last_error().
void set_last_error(const char* msg);

// Options of the tensor-core indexer used by the fused indexer -> top-k.
struct IndexerExtra {
  int kstride = 1;        // score key tiles 0, kstride, 2*kstride, ... only (a sample)
  long long ldT = 0;      // output row length in floats (0: T); tile kt -> columns kt*128..
  const uint32_t* tau = nullptr;  // filter mode: per-row order-key thresholds [B*S]
  uint2* cand = nullptr;          // [B*S, cand_cap] candidates: (order key, key position)
  int* cand_cnt = nullptr;        // [B*S] candidates found (may exceed cand_cap), zeroed
  int cand_cap = 0;
  const int* run_if = nullptr;    // device flag: the launch does nothing while it is 0
};

// Indexer scores, SIMT (float32 FMA) kernel: any dtype, DI <= 128.
cudaError_t launch_index_scores_simt(int dtype, const void* q_idx, const void* k_idx,
                                     const float* w, float scale, int relu, int B, int S,
                                     int T, int HI, int DI, int q_off, float* scores,
                                     cudaStream_t st);


// Indexer scores on the tensor cores (tcgen05 + TMEM + TMA): bf16, DI in {64,128,...}.
// Returns cudaErrorNotSupported for shapes it does not take.
bool index_scores_tc_supported(int dtype, int HI, int DI);
cudaError_t launch_index_scores_tc(const void* q_idx, const void* k_idx, const float* w,
                                   float scale, int relu, int B, int S, int T, int HI, int DI,
                                   int q_off, float* scores, int write_masked,
                                   cudaStream_t st, const IndexerExtra* ex = nullptr);

// Indexer scores with e4m3 operands (tcgen05 kind::f8f6f4): HI in {16, 32}, DI == 128.
bool index_scores_e4m3_supported(int HI, int DI);
cudaError_t launch_index_scores_e4m3(const void* q_idx, const void* k_idx, const float* w,
                                     float scale, int relu, int B, int S, int T, int HI, int DI,
                                     int q_off, float* scores, int write_masked,
                                     cudaStream_t st);

// Head-collapsed indexer (valid when no ReLU is applied per head: the score is linear in
// q_I): launch_collapse_q writes qc [rows, 2, DI] bf16 (hi and lo parts of
// sum_h w[s,h] q_I[s,h,:]); launch_index_scores_collapsed scores k_I against them on the
// tensor cores.  bf16, DI in {64, 128}, relu != per-head.
bool index_scores_collapsed_supported(int dtype, int DI, int relu);
cudaError_t launch_collapse_q(const void* q_idx, const float* w, long long rows, int HI, int DI,
                              void* qc, cudaStream_t st);
cudaError_t launch_index_scores_collapsed(const void* qc, const void* k_idx, float scale,
                                          int relu, int B, int S, int T, int DI, int q_off,
                                          float* scores, int write_masked, cudaStream_t st,
                                          const IndexerExtra* ex = nullptr);

// Hadamard rotation of indexer inputs: out[r] = x[r] @ H / sqrt(d), d in {64, 128};
// dtype 0 float32, 1 bf16; out may equal x.
cudaError_t launch_hadamard(int dtype, const void* x, void* out, long long rows, int d,
                            cudaStream_t st);

// Per-row top-k (radix select + ordered compaction).  `mask` (optional) receives the
// selection bitmask, one bit per key, rows of `mask_stride` 32-bit words
// (mask_stride >= ceil(T/32); words past the row's keys are zero).
// The lower bound of bucket b of the top-k's 12-bit key prefix as a float (the host build of
// the function its second read compares scores against; testing aid).
float topk_bucket_floor(unsigned b);
cudaError_t launch_topk(const float* scores, int B, int S, int T, int K, int q_off,
                        int32_t* idx, uint32_t* mask, int mask_stride, cudaStream_t st,
                        const int* run_if = nullptr);
// Fused indexer -> top-k, after the sampled indexer pass: tau[row] = the order key of the
// r-th largest sampled score (0, i.e. keep everything, for rows of at most `cap` keys).
cudaError_t launch_topk_tau(const float* sample, long long ld, int B, int S, int T, int K,
                            int q_off, int kstride, int cap, uint32_t* tau, cudaStream_t st);
// ... and after the filtered indexer pass: the exact top-k of every row from its candidate
// list, or *fail = 1 when some row's list cannot hold it (< K or > cap candidates).
size_t topk_candidates_smem(int T, int cap);
cudaError_t launch_topk_candidates(const uint2* cand, const int* cand_cnt, int cap, int B,
                                   int S, int T, int K,
                                   int q_off, int32_t* idx, uint32_t* mask, int mask_stride,
                                   int* fail, cudaStream_t st);
// Selection bitmask from index lists (valid, causal entries only).
cudaError_t launch_idx_to_mask(const int32_t* idx, int B, int S, int T, int K, int q_off,
                               uint32_t* mask, int mask_stride, cudaStream_t st);
// Words per bitmask row used by the masked-tile attention (ceil(T/128) * 4).
inline int mask_stride_words(int T) { return ((T + 127) / 128) * 4; }
// The masked-tile attention's workspace: the selection mask rows, then (256-byte aligned) its
// block list -- per (batch row, block of 128 queries) the number of key blocks (of 128 keys)
// any of its queries selected from, [B * nqb] int32, and those blocks in ascending order,
// [B * nqb, nkb] uint16.
inline size_t masked_attn_mask_bytes(int B, int S, int T) {
  const size_t m = ((size_t)B * S * mask_stride_words(T) * 4 + 255) & ~(size_t)255;
  const size_t nqb = (size_t)((S + 127) / 128), nkb = (size_t)((T + 127) / 128);
  return m + (size_t)B * nqb * 4 + (size_t)B * nqb * nkb * 2;
}
inline void* masked_attn_blocks(uint32_t* mask, int B, int S, int T) {
  return reinterpret_cast<uint8_t*>(mask) +
         (((size_t)B * S * mask_stride_words(T) * 4 + 255) & ~(size_t)255);
}

// Gather attention (idx lists) and band attention (sliding window, GQA) share one kernel.
struct AttnProblem {
  int dtype;          // 0 f32, 1 bf16
  const void* q;      // [B,S,H,DQK]
  const void* k;      // [B,T,HKV,DQK]
  const void* v;      // [B,T,HKV,DV]
  const int32_t* idx; // [B,S,K] or NULL for the band
  int K;              // idx columns
  int window;         // band width when idx == NULL
  const void* gate;   // [B,S,H] or NULL
  int gate_mode;
  float sm_scale;
  int B, S, T, H, HKV, DQK, DV, q_off;
  void* out;          // [B,S,H,DV]
  const void* sink_k = nullptr;  // [nsink,HKV,DQK] attention sinks (PAS), or NULL
  const void* sink_v = nullptr;  // [nsink,HKV,DV]
  int nsink = 0;
};
size_t gather_attn_workspace_bytes(int B, int S, int H, int DV, int K, int nsink = 0);
// Testing aid: the next launch_gather_attn makes its first CTA fill none of its key slots,
// so that CTA's bounded waits run out and record the timeout (one-shot).
void arm_gather_skip_copy();
cudaError_t launch_gather_attn(const AttnProblem& p, void* ws, size_t ws_bytes,
                               cudaStream_t st);

// Dense tensor-core attention tiles under the selection bitmask (or, with idx == NULL and
// mask == NULL, under the sliding-window band).  bf16, DQK in {128, 192}, DV == 128.
bool masked_attn_supported(int dtype, int DQK, int DV);
// With a mask, `blocks` (masked_attn_blocks of the mask buffer) receives the block list first,
// and key blocks no query of a 128-query block selected are skipped.
cudaError_t launch_masked_attn(const AttnProblem& p, const uint32_t* mask, int mask_stride,
                               void* blocks, cudaStream_t st);

// Merge of split-key partials (unnormalised o [rows, nsplit, H, DV] float32 and (m, l)
// [rows, nsplit, H, 2], m in log2 units) into out [rows, H, DV], gate applied.  nsplit <= 64.
cudaError_t launch_split_combine(int dtype, const float* part_o, const float* part_ml, int rows,
                                 int nsplit, int H, int DV, const void* gate, int gate_mode,
                                 void* out, cudaStream_t st);

// Sparse attention over a shared latent cache (MQA form): q [B,S,H,576], kv [B,T,576] (keys =
// whole rows, values = their first 512 dims), bf16, 1 <= H <= 128.
struct LatentProblem {
  int dtype;
  const void* q;
  const void* kv;
  const int32_t* idx;  // [B,S,K]
  int K;
  const void* sink;    // [nsink, 576] latent sink rows (PAS) or NULL
  int nsink;
  const void* gate;    // [B,S,H] or NULL
  int gate_mode;
  float sm_scale;
  int B, S, T, H, DQK, DV, q_off;
  void* out;           // [B,S,H,DV]
};
bool latent_attn_supported(int dtype, int H, int DQK, int DV);
size_t latent_attn_workspace_bytes(int B, int S, int H, int K, int nsink);
cudaError_t launch_latent_attn(const LatentProblem& p, void* ws, size_t ws_bytes,
                               cudaStream_t st);

}  // namespace dsa
