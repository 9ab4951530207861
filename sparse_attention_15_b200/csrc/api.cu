// libdsa C ABI: argument validation, workspace layout and kernel dispatch.
// The contract of every entry point is documented in include/dsa.h.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>

#include <mutex>
#include <string>
#include <vector>

#include "../../include/dsa.h"
#include "checks.h"
#include "common.cuh"
#include "kernels.h"

namespace dsa {
namespace {
std::mutex g_status_mu;
std::vector<const void*>& status_words() {
  static std::vector<const void*> words;
  return words;
}
}  // namespace
void register_status_word(const void* symbol) {
  std::lock_guard<std::mutex> lk(g_status_mu);
  status_words().push_back(symbol);
}
}  // namespace dsa

namespace {

thread_local std::string g_last_error;

dsa_status fail(dsa_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

dsa_status cuda_status(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return DSA_OK;
  if (e == cudaErrorNotSupported)
    return fail(DSA_ERR_UNSUPPORTED, "%s: no kernel for this shape", what);
  return fail(DSA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t esize(dsa_dtype dt) { return dt == DSA_F32 ? 4 : (dt == DSA_E4M3 ? 1 : 2); }

bool dim_ok(dsa_dtype dt, int d) { return d > 0 && d % (dt == DSA_F32 ? 4 : 8) == 0; }

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

#define REQUIRE(cond, st, ...)                 \
  do {                                         \
    if (!(cond)) return fail(st, __VA_ARGS__); \
  } while (0)

dsa_status check_index_args(dsa_dtype dtype, const void* q_idx, const void* k_idx,
                            const float* w, float scale, dsa_relu_mode relu, int B, int S,
                            int T, int HI, int DI, const void* scores) {
  REQUIRE(dtype == DSA_F32 || dtype == DSA_BF16 || dtype == DSA_E4M3, DSA_ERR_INVALID_ARG,
          "unknown dtype %d", (int)dtype);
  REQUIRE(q_idx && k_idx && w && scores, DSA_ERR_INVALID_ARG, "null pointer argument");
  REQUIRE(B > 0 && S > 0 && T > 0 && HI > 0 && DI > 0, DSA_ERR_INVALID_ARG,
          "sizes must be positive (B=%d S=%d T=%d HI=%d DI=%d)", B, S, T, HI, DI);
  REQUIRE(T >= S, DSA_ERR_INVALID_ARG, "T (%d) must be >= S (%d): queries are the last S keys",
          T, S);
  REQUIRE(isfinite(scale) && scale > 0.f, DSA_ERR_INVALID_ARG,
          "index scale must be finite and > 0");
  REQUIRE(relu >= DSA_RELU_NONE && relu <= DSA_RELU_PER_HEAD, DSA_ERR_INVALID_ARG,
          "unknown relu mode %d", (int)relu);
  REQUIRE(HI <= 256, DSA_ERR_UNSUPPORTED, "HI=%d > 256", HI);
  REQUIRE(DI <= 128 && dim_ok(dtype, DI), DSA_ERR_UNSUPPORTED,
          "DI=%d must be <= 128 and a multiple of %d", DI, dtype == DSA_F32 ? 4 : 8);
  REQUIRE(dtype != DSA_E4M3 || dsa::index_scores_e4m3_supported(HI, DI), DSA_ERR_UNSUPPORTED,
          "e4m3 indexer inputs need HI in {16,32} and DI == 128 (HI=%d DI=%d)", HI, DI);
  REQUIRE(S <= 65535 * 8, DSA_ERR_UNSUPPORTED, "S=%d too large", S);
  REQUIRE(B <= 65535, DSA_ERR_UNSUPPORTED, "B=%d too large", B);
  REQUIRE(aligned16(q_idx) && aligned16(k_idx) && aligned16(w) && aligned16(scores),
          DSA_ERR_UNSUPPORTED, "pointers must be 16-byte aligned");
  return DSA_OK;
}

dsa_status run_index_scores(dsa_dtype dtype, const void* q_idx, const void* k_idx,
                            const float* w, float scale, dsa_relu_mode relu, int B, int S,
                            int T, int HI, int DI, int q_off, float* scores, int write_masked,
                            cudaStream_t st) {
  cudaError_t e;
  if (dtype == DSA_E4M3)
    e = dsa::launch_index_scores_e4m3(q_idx, k_idx, w, scale, (int)relu, B, S, T, HI, DI, q_off,
                                      scores, write_masked, st);
  else if (dsa::index_scores_tc_supported((int)dtype, HI, DI))
    e = dsa::launch_index_scores_tc(q_idx, k_idx, w, scale, (int)relu, B, S, T, HI, DI, q_off,
                                    scores, write_masked, st);
  else
    e = dsa::launch_index_scores_simt((int)dtype, q_idx, k_idx, w, scale, (int)relu, B, S, T,
                                      HI, DI, q_off, scores, st);
  return cuda_status(e, "dsa_index_scores");
}

size_t collapsed_q_bytes(int B, int S, int DI) {
  return (size_t)B * S * 2 * DI * sizeof(uint16_t);
}

dsa_status check_collapsed(dsa_dtype dtype, dsa_relu_mode relu, int DI) {
  REQUIRE(dsa::index_scores_collapsed_supported((int)dtype, DI, (int)relu), DSA_ERR_UNSUPPORTED,
          "the collapsed indexer needs bf16, DI in {64,128} and no per-head ReLU");
  return DSA_OK;
}

// qc for rows [0, B*S) (q_idx/w as given), then the collapsed scores of B x S queries.
dsa_status run_collapse_q(const void* q_idx, const float* w, long long rows, int HI, int DI,
                          void* qc, cudaStream_t st) {
  return cuda_status(dsa::launch_collapse_q(q_idx, w, rows, HI, DI, qc, st),
                     "collapse_q");
}

dsa_status run_index_scores_collapsed(const void* qc, const void* k_idx, float scale,
                                      dsa_relu_mode relu, int B, int S, int T, int DI, int q_off,
                                      float* scores, int write_masked, cudaStream_t st) {
  return cuda_status(dsa::launch_index_scores_collapsed(qc, k_idx, scale, (int)relu, B, S, T, DI,
                                                        q_off, scores, write_masked, st),
                     "dsa_index_scores_collapsed");
}

// ----------------------------------------------------------------------------- fused
// Workspace of the fused indexer -> top-k (section 2b of dsa.h): the sampled scores, the
// thresholds, the candidate counters (+ the fallback flag), the candidate lists and the
// full score matrix the fallback uses.
struct FusedLayout {
  int kstride, cap;
  long long ld;  // sampled columns per row
  size_t qc_off, sample_off, tau_off, cnt_off, cand_off, scores_off, total;
};

FusedLayout fused_layout(int B, int S, int T, int K_eff) {
  FusedLayout L{};
  const int ntiles = (T + 127) / 128;
  L.kstride = ntiles / 32 > 4 ? ntiles / 32 : 4;
  L.cap = 2 * K_eff + 1024;
  L.ld = (long long)(((ntiles - 1) / L.kstride) + 1) * 128;
  const size_t rows = (size_t)B * S;
  size_t off = 0;
  L.qc_off = off;     off += align256(rows * 2 * 128 * sizeof(uint16_t));  // collapsed q_I
  L.sample_off = off; off += align256(rows * (size_t)L.ld * sizeof(float));
  L.tau_off = off;    off += align256(rows * sizeof(uint32_t));
  L.cnt_off = off;    off += align256((rows + 1) * sizeof(int));  // + the fallback flag
  L.cand_off = off;   off += align256(rows * (size_t)L.cap * sizeof(uint2));
  L.scores_off = off; off += align256(rows * (size_t)T * sizeof(float));
  L.total = off;
  return L;
}

bool fused_supported(dsa_dtype dtype, int HI, int DI, int T, int K_eff) {
  return dsa::index_scores_tc_supported((int)dtype, HI, DI) &&
         dsa::topk_candidates_smem(T, 2 * K_eff + 1024) <= 220u * 1024u;
}

// Enqueues the fused indexer -> top-k into ws (laid out by fused_layout): idx (and the
// selection mask, if given) for every row; *fallback_out (optional) = whether the
// full-score path ran.
dsa_status run_fused_index_topk(const void* q_idx, const void* k_idx, const float* w,
                                float scale, dsa_relu_mode relu, int B, int S, int T, int HI,
                                int DI, int K_eff, int32_t* idx, uint32_t* mask,
                                int mask_stride, uint8_t* ws, int32_t* fallback_out,
                                cudaStream_t st, cudaEvent_t after_indexer) {
  const FusedLayout L = fused_layout(B, S, T, K_eff);
  const int q_off = T - S;
  const size_t rows = (size_t)B * S;
  float* sample = reinterpret_cast<float*>(ws + L.sample_off);
  uint32_t* tau = reinterpret_cast<uint32_t*>(ws + L.tau_off);
  int* cnt = reinterpret_cast<int*>(ws + L.cnt_off);
  int* fail = cnt + rows;
  uint2* cand = reinterpret_cast<uint2*>(ws + L.cand_off);
  float* scores = reinterpret_cast<float*>(ws + L.scores_off);
  cudaError_t e = cudaMemsetAsync(cnt, 0, (rows + 1) * sizeof(int), st);
  if (e != cudaSuccess) return cuda_status(e, "fused/clear");
  // 1. the sample: every kstride-th key tile of each row.  Without a per-head ReLU the score
  // is linear in q_I and the head-collapsed indexer gives the same scores (exactly for
  // integer inputs, to float32 rounding of its hi/lo split otherwise) for 1/HI of the work;
  // the threshold only steers how many candidates pass, the count check keeps it exact
  dsa::IndexerExtra xs{};
  xs.kstride = L.kstride;
  xs.ldT = L.ld;
  if (dsa::index_scores_collapsed_supported(1, DI, (int)relu)) {
    void* qc = ws + L.qc_off;
    e = dsa::launch_collapse_q(q_idx, w, (long long)rows, HI, DI, qc, st);
    if (e == cudaSuccess)
      e = dsa::launch_index_scores_collapsed(qc, k_idx, scale, (int)relu, B, S, T, DI, q_off,
                                             sample, 0, st, &xs);
  } else {
    e = dsa::launch_index_scores_tc(q_idx, k_idx, w, scale, (int)relu, B, S, T, HI, DI, q_off,
                                    sample, 0, st, &xs);
  }
  if (e != cudaSuccess) return cuda_status(e, "fused/sample");
  // 2. the thresholds
  e = dsa::launch_topk_tau(sample, L.ld, B, S, T, K_eff, q_off, L.kstride, L.cap, tau, st);
  if (e != cudaSuccess) return cuda_status(e, "fused/tau");
  // 3. every score, kept only as a candidate when it reaches its row's threshold
  dsa::IndexerExtra xf{};
  xf.tau = tau; xf.cand = cand; xf.cand_cnt = cnt; xf.cand_cap = L.cap;
  e = dsa::launch_index_scores_tc(q_idx, k_idx, w, scale, (int)relu, B, S, T, HI, DI, q_off,
                                  nullptr, 0, st, &xf);
  if (e != cudaSuccess) return cuda_status(e, "fused/filter");
  if (after_indexer && (e = cudaEventRecord(after_indexer, st)) != cudaSuccess)
    return cuda_status(e, "fused/event");
  // 4. the exact top-k of every row from its candidates (or the fallback flag)
  e = dsa::launch_topk_candidates(cand, cnt, L.cap, B, S, T, K_eff, q_off, idx, mask,
                                  mask_stride, fail, st);
  if (e != cudaSuccess) return cuda_status(e, "fused/select");
  // 5. the fallback, a no-op unless some row raised the flag: full scores, full top-k
  dsa::IndexerExtra xr{};
  xr.run_if = fail;
  e = dsa::launch_index_scores_tc(q_idx, k_idx, w, scale, (int)relu, B, S, T, HI, DI, q_off,
                                  scores, 0, st, &xr);
  if (e != cudaSuccess) return cuda_status(e, "fused/fallback scores");
  e = dsa::launch_topk(scores, B, S, T, K_eff, q_off, idx, mask, mask_stride, st, fail);
  if (e != cudaSuccess) return cuda_status(e, "fused/fallback top-k");
  if (fallback_out &&
      (e = cudaMemcpyAsync(fallback_out, fail, sizeof(int), cudaMemcpyDeviceToDevice, st)) !=
          cudaSuccess)
    return cuda_status(e, "fused/fallback flag");
  return DSA_OK;
}

// Attention sinks ([PANGU] §3.4 PAS): up to one 128-entry block, [nsink, H, D] rows.
dsa_status check_sinks(const void* sink_k, const void* sink_v, int nsink) {
  if (nsink == 0) return DSA_OK;
  REQUIRE(nsink > 0 && nsink <= 128, DSA_ERR_UNSUPPORTED, "nsink=%d must be in [1, 128]",
          nsink);
  REQUIRE(sink_k != nullptr && sink_v != nullptr, DSA_ERR_INVALID_ARG,
          "sink_k and sink_v must be given with nsink > 0");
  REQUIRE(aligned16(sink_k) && aligned16(sink_v), DSA_ERR_UNSUPPORTED,
          "sink pointers must be 16-byte aligned");
  return DSA_OK;
}


float default_scale(float sm_scale, int DQK) {
  return sm_scale > 0.f ? sm_scale : 1.0f / sqrtf((float)DQK);
}

constexpr int kNone = -1, kGather = 1, kMasked = 2, kLatent = 3;

size_t mask_bytes(int B, int S, int T) { return dsa::masked_attn_mask_bytes(B, S, T); }

// Cost model of the two attention algorithms.  Gather: every selected (query, key) pair
// moves one K row and one V row (H * (DQK + DV) elements).  Masked tile: every 128-query
// block runs dense tiles over all its causal 128-key blocks, 4 * H * (DQK + DV) flops per
// executed pair.  Rates: a sustained gather bandwidth of 4 TB/s and half the bf16 tensor
// peak; only their ratio matters.
int choose_algo(dsa_attn_algo req, dsa_dtype dt, int B, int S, int T, int H, int DQK, int DV,
                int K) {
  const bool tc = dsa::masked_attn_supported((int)dt, DQK, DV);
  if (req == DSA_ATTN_GATHER) return kGather;
  if (req == DSA_ATTN_MASKED_TILE) return tc ? kMasked : kNone;
  if (!tc) return kGather;
  const long long q_off = (long long)T - S;
  double dense = 0.0, sel = 0.0;
  for (long long s0 = 0; s0 < S; s0 += 128) {
    const long long s_last = (S - 1 < s0 + 127) ? S - 1 : s0 + 127;
    const long long t_hi = (T - 1 < s_last + q_off) ? T - 1 : s_last + q_off;
    dense += 128.0 * (double)((t_hi / 128 + 1) * 128);
  }
  for (long long s = 0; s < S; ++s) {
    const long long n = (s + q_off + 1 < T) ? s + q_off + 1 : T;
    sel += (double)(n < K ? n : K);
  }
  const double per_pair = (double)H * (DQK + DV);
  const double t_dense = B * dense * per_pair * 2.0 / 0.8e15;
  const double t_gather = B * sel * per_pair * 2.0 / 4.0e12;
  return t_dense < t_gather ? kMasked : kGather;
}

}  // namespace

namespace dsa {
// Records the thread-local text dsa_last_error() returns (for entry points in other files).
void set_last_error(const char* msg) { g_last_error = msg ? msg : ""; }

// Argument checks shared by the attention entry points (declared in checks.h).
dsa_status check_attn_common(dsa_dtype dtype, const void* q, const void* k, const void* v,
                             const void* gate, dsa_gate_mode gm, float sm_scale, int B, int S,
                             int T, int H, int HKV, int DQK, int DV, const void* out) {
  REQUIRE(dtype == DSA_F32 || dtype == DSA_BF16, DSA_ERR_INVALID_ARG, "unknown dtype %d",
          (int)dtype);
  REQUIRE(q && k && v && out, DSA_ERR_INVALID_ARG, "null pointer argument");
  REQUIRE(B > 0 && S > 0 && T > 0 && H > 0 && HKV > 0 && DQK > 0 && DV > 0,
          DSA_ERR_INVALID_ARG, "sizes must be positive");
  REQUIRE(T >= S, DSA_ERR_INVALID_ARG, "T (%d) must be >= S (%d)", T, S);
  REQUIRE(H % HKV == 0, DSA_ERR_INVALID_ARG, "H=%d not a multiple of HKV=%d", H, HKV);
  REQUIRE(gm >= DSA_GATE_OFF && gm <= DSA_GATE_SILU, DSA_ERR_INVALID_ARG,
          "unknown gate mode %d (only sigmoid and silu exist)", (int)gm);
  REQUIRE((gm == DSA_GATE_OFF) == (gate == nullptr), DSA_ERR_INVALID_ARG,
          "gate pointer must be given exactly when the gate is on");
  REQUIRE(!isnan(sm_scale) && !isinf(sm_scale), DSA_ERR_INVALID_ARG, "sm_scale not finite");
  REQUIRE(DQK <= 256 && DV <= 256 && dim_ok(dtype, DQK) && dim_ok(dtype, DV),
          DSA_ERR_UNSUPPORTED, "DQK=%d / DV=%d must be <= 256 and multiples of %d", DQK, DV,
          dtype == DSA_F32 ? 4 : 8);
  REQUIRE(H <= 64, DSA_ERR_UNSUPPORTED, "H=%d > 64", H);
  REQUIRE((HKV * DQK * esize(dtype)) % 16 == 0 && (HKV * DV * esize(dtype)) % 16 == 0,
          DSA_ERR_UNSUPPORTED, "K/V rows must be multiples of 16 bytes");
  REQUIRE(aligned16(q) && aligned16(k) && aligned16(v) && aligned16(out) &&
              (gate == nullptr || aligned16(gate)),
          DSA_ERR_UNSUPPORTED, "pointers must be 16-byte aligned");
  return DSA_OK;
}

dsa_status check_idx_args(const int32_t* idx, int K) {
  REQUIRE(idx != nullptr && K > 0, DSA_ERR_INVALID_ARG, "idx must be given with K > 0");
  REQUIRE(aligned16(idx), DSA_ERR_UNSUPPORTED, "idx must be 16-byte aligned");
  return DSA_OK;
}
}  // namespace dsa

extern "C" {

const char* dsa_status_string(dsa_status s) {
  switch (s) {
    case DSA_OK: return "ok";
    case DSA_ERR_INVALID_ARG: return "invalid argument";
    case DSA_ERR_UNSUPPORTED: return "unsupported shape or layout";
    case DSA_ERR_CUDA: return "CUDA error";
    case DSA_ERR_TIMEOUT: return "in-kernel wait timed out";
    case DSA_ERR_INTERNAL: return "internal consistency check failed";
  }
  return "unknown status";
}

const char* dsa_last_error(void) { return g_last_error.c_str(); }

const char* dsa_version(void) { return "dsa-b200 0.2.0 sm_100a"; }

float dsa_test_topk_bucket_floor(unsigned b) { return dsa::topk_bucket_floor(b); }

dsa_status dsa_test_arm_wait_timeout(void) {
  dsa::arm_gather_skip_copy();
  return DSA_OK;
}

dsa_status dsa_device_status(int reset) {
  std::vector<const void*> words;
  {
    std::lock_guard<std::mutex> lk(dsa::g_status_mu);
    words = dsa::status_words();
  }
  unsigned v = 0;
  for (const void* sym : words) {  // every source file's word
    unsigned w = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&w, sym, sizeof(w));
    if (e != cudaSuccess)
      return fail(DSA_ERR_CUDA, "dsa_device_status: %s", cudaGetErrorString(e));
    if (reset && w) {
      const unsigned z = 0;
      e = cudaMemcpyToSymbol(sym, &z, sizeof(z));
      if (e != cudaSuccess)
        return fail(DSA_ERR_CUDA, "dsa_device_status: %s", cudaGetErrorString(e));
    }
    v |= w;
  }
  if (v & dsa::kStatusTimeout) return fail(DSA_ERR_TIMEOUT, "an in-kernel wait timed out");
  if (v & dsa::kStatusInternal) return fail(DSA_ERR_INTERNAL, "in-kernel check failed");
  return DSA_OK;
}

dsa_status dsa_index_scores(dsa_dtype dtype, const void* q_idx, const void* k_idx,
                            const float* w, float scale, dsa_relu_mode relu, int B, int S,
                            int T, int HI, int DI, float* scores, dsa_stream_t stream) {
  dsa_status st = check_index_args(dtype, q_idx, k_idx, w, scale, relu, B, S, T, HI, DI, scores);
  if (st != DSA_OK) return st;
  return run_index_scores(dtype, q_idx, k_idx, w, scale, relu, B, S, T, HI, DI, T - S, scores,
                          1, (cudaStream_t)stream);
}

size_t dsa_index_scores_collapsed_workspace_bytes(int B, int S, int DI) {
  if (B <= 0 || S <= 0 || DI <= 0) return 0;
  return collapsed_q_bytes(B, S, DI);
}

dsa_status dsa_index_scores_collapsed(dsa_dtype dtype, const void* q_idx, const void* k_idx,
                                      const float* w, float scale, dsa_relu_mode relu, int B,
                                      int S, int T, int HI, int DI, float* scores, void* ws,
                                      size_t ws_bytes, dsa_stream_t stream) {
  dsa_status st = check_index_args(dtype, q_idx, k_idx, w, scale, relu, B, S, T, HI, DI, scores);
  if (st != DSA_OK) return st;
  if ((st = check_collapsed(dtype, relu, DI)) != DSA_OK) return st;
  REQUIRE(ws != nullptr && ws_bytes >= collapsed_q_bytes(B, S, DI), DSA_ERR_INVALID_ARG,
          "workspace too small: %zu bytes given, %zu needed", ws_bytes,
          collapsed_q_bytes(B, S, DI));
  REQUIRE(aligned16(ws), DSA_ERR_UNSUPPORTED, "workspace must be 16-byte aligned");
  cudaStream_t s = (cudaStream_t)stream;
  if ((st = run_collapse_q(q_idx, w, (long long)B * S, HI, DI, ws, s)) != DSA_OK) return st;
  return run_index_scores_collapsed(ws, k_idx, scale, relu, B, S, T, DI, T - S, scores, 1, s);
}

dsa_status dsa_hadamard_rotate(dsa_dtype dtype, const void* x, long long rows, int d, void* out,
                               dsa_stream_t stream) {
  REQUIRE(dtype == DSA_F32 || dtype == DSA_BF16, DSA_ERR_UNSUPPORTED,
          "the rotation takes float32 or bf16 (dtype %d)", (int)dtype);
  REQUIRE(x && out, DSA_ERR_INVALID_ARG, "null pointer argument");
  REQUIRE(rows > 0, DSA_ERR_INVALID_ARG, "rows must be positive");
  REQUIRE(d == 64 || d == 128, DSA_ERR_UNSUPPORTED, "d=%d must be 64 or 128", d);
  REQUIRE(aligned16(x) && aligned16(out), DSA_ERR_UNSUPPORTED, "pointers must be 16-byte aligned");
  return cuda_status(dsa::launch_hadamard((int)dtype, x, out, rows, d, (cudaStream_t)stream),
                     "dsa_hadamard_rotate");
}

dsa_status dsa_topk(const float* scores, int B, int S, int T, int K, int32_t* idx,
                    dsa_stream_t stream) {
  REQUIRE(scores && idx, DSA_ERR_INVALID_ARG, "null pointer argument");
  REQUIRE(B > 0 && S > 0 && T > 0 && K > 0, DSA_ERR_INVALID_ARG, "sizes must be positive");
  REQUIRE(T >= S, DSA_ERR_INVALID_ARG, "T (%d) must be >= S (%d)", T, S);
  REQUIRE((size_t)B * S <= 0x7fffffffu, DSA_ERR_UNSUPPORTED, "too many rows");
  REQUIRE(aligned16(scores) && aligned16(idx), DSA_ERR_UNSUPPORTED,
          "pointers must be 16-byte aligned");
  return cuda_status(dsa::launch_topk(scores, B, S, T, K, T - S, idx, nullptr, 0,
                                      (cudaStream_t)stream),
                     "dsa_topk");
}

size_t dsa_index_topk_workspace_bytes(int B, int S, int T, int K) {
  if (B <= 0 || S <= 0 || T <= 0 || K <= 0) return 0;
  return fused_layout(B, S, T, K < T ? K : T).total;
}

dsa_status dsa_index_topk(dsa_dtype dtype, const void* q_idx, const void* k_idx,
                          const float* w, float scale, dsa_relu_mode relu, int B, int S, int T,
                          int HI, int DI, int K, int32_t* idx, void* ws, size_t ws_bytes,
                          int32_t* fallback_out, dsa_stream_t stream) {
  dsa_status st = check_index_args(dtype, q_idx, k_idx, w, scale, relu, B, S, T, HI, DI, idx);
  if (st != DSA_OK) return st;
  REQUIRE(K > 0, DSA_ERR_INVALID_ARG, "K must be positive");
  REQUIRE((size_t)B * S <= 0x7fffffffu, DSA_ERR_UNSUPPORTED, "too many rows");
  const int k_eff = K < T ? K : T;
  REQUIRE(fused_supported(dtype, HI, DI, T, k_eff), DSA_ERR_UNSUPPORTED,
          "the fused indexer -> top-k needs bf16 inputs, HI in {16,32}, DI in {64,128} and "
          "T, K small enough for the candidate select (T=%d, K=%d)", T, k_eff);
  const size_t need = fused_layout(B, S, T, k_eff).total;
  REQUIRE(ws != nullptr && ws_bytes >= need, DSA_ERR_INVALID_ARG,
          "workspace too small: %zu bytes given, %zu needed", ws_bytes, need);
  REQUIRE(aligned16(ws) && (fallback_out == nullptr || aligned16(fallback_out)),
          DSA_ERR_UNSUPPORTED, "workspace and fallback_out must be 16-byte aligned");
  return run_fused_index_topk(q_idx, k_idx, w, scale, relu, B, S, T, HI, DI, k_eff, idx,
                              nullptr, 0, static_cast<uint8_t*>(ws), fallback_out,
                              (cudaStream_t)stream, nullptr);
}

size_t dsa_sparse_attn_workspace_bytes(dsa_dtype dtype, int B, int S, int T, int H, int DQK,
                                       int DV, int K, dsa_attn_algo algo) {
  return dsa_sparse_attn_sinks_workspace_bytes(dtype, B, S, T, H, DQK, DV, K, 0, algo);
}

size_t dsa_sparse_attn_sinks_workspace_bytes(dsa_dtype dtype, int B, int S, int T, int H,
                                             int DQK, int DV, int K, int nsink,
                                             dsa_attn_algo algo) {
  if (B <= 0 || S <= 0 || T <= 0 || H <= 0 || DQK <= 0 || DV <= 0 || K <= 0 || nsink < 0)
    return 0;
  const int alg = choose_algo(algo, dtype, B, S, T, H, DQK, DV, K);
  if (alg == kMasked) return mask_bytes(B, S, T);
  if (alg == kGather) return dsa::gather_attn_workspace_bytes(B, S, H, DV, K, nsink);
  return 0;
}

dsa_attn_algo dsa_sparse_attn_algo(dsa_dtype dtype, int B, int S, int T, int H, int DQK, int DV,
                                   int K, dsa_attn_algo algo) {
  if (B <= 0 || S <= 0 || T <= 0 || H <= 0 || DQK <= 0 || DV <= 0 || K <= 0) return DSA_ATTN_AUTO;
  const int alg = choose_algo(algo, dtype, B, S, T, H, DQK, DV, K);
  return alg == kMasked ? DSA_ATTN_MASKED_TILE : (alg == kGather ? DSA_ATTN_GATHER : DSA_ATTN_AUTO);
}

// Latent (MQA-form) attention: bf16, DQK 576 / DV 512, 1 <= H <= 128, latent sink rows.
static dsa_status check_latent(dsa_dtype dtype, const void* q, const void* kv,
                               const void* sink_kv, int nsink, const void* gate,
                               dsa_gate_mode gm, float sm_scale, int B, int S, int T, int H,
                               int DQK, int DV, const void* out) {
  REQUIRE(dtype == DSA_F32 || dtype == DSA_BF16, DSA_ERR_INVALID_ARG, "unknown dtype %d",
          (int)dtype);
  REQUIRE(q && kv && out, DSA_ERR_INVALID_ARG, "null pointer argument");
  REQUIRE(B > 0 && S > 0 && T > 0 && H > 0 && DQK > 0 && DV > 0, DSA_ERR_INVALID_ARG,
          "sizes must be positive");
  REQUIRE(T >= S, DSA_ERR_INVALID_ARG, "T (%d) must be >= S (%d)", T, S);
  REQUIRE(DV <= DQK, DSA_ERR_INVALID_ARG, "DV=%d exceeds the latent row (DQK=%d)", DV, DQK);
  REQUIRE(gm >= DSA_GATE_OFF && gm <= DSA_GATE_SILU, DSA_ERR_INVALID_ARG,
          "unknown gate mode %d (only sigmoid and silu exist)", (int)gm);
  REQUIRE((gm == DSA_GATE_OFF) == (gate == nullptr), DSA_ERR_INVALID_ARG,
          "gate pointer must be given exactly when the gate is on");
  REQUIRE(!isnan(sm_scale) && !isinf(sm_scale), DSA_ERR_INVALID_ARG, "sm_scale not finite");
  REQUIRE(nsink >= 0 && nsink <= 128, DSA_ERR_UNSUPPORTED, "nsink=%d must be in [0, 128]",
          nsink);
  REQUIRE((nsink > 0) == (sink_kv != nullptr), DSA_ERR_INVALID_ARG,
          "sink_kv must be given exactly when nsink > 0");
  REQUIRE(dsa::latent_attn_supported((int)dtype, H, DQK, DV), DSA_ERR_UNSUPPORTED,
          "latent attention needs bf16, DQK == 576, DV == 512 and 1 <= H <= 128");
  REQUIRE((long long)B * S * 128 <= 0x7fffffffLL, DSA_ERR_UNSUPPORTED, "B*S=%lld too large",
          (long long)B * S);
  REQUIRE(aligned16(q) && aligned16(kv) && aligned16(out) &&
              (gate == nullptr || aligned16(gate)) && (sink_kv == nullptr || aligned16(sink_kv)),
          DSA_ERR_UNSUPPORTED, "pointers must be 16-byte aligned");
  return DSA_OK;
}

static dsa::LatentProblem latent_problem(const void* q, const void* kv, const int32_t* idx, int K,
                                         const void* sink_kv, int nsink, const void* gate,
                                         dsa_gate_mode gm, float sm_scale, int B, int S, int T,
                                         int H, int DQK, int DV, void* out) {
  dsa::LatentProblem p{};
  p.dtype = (int)DSA_BF16; p.q = q; p.kv = kv; p.idx = idx; p.K = K;
  p.sink = nsink > 0 ? sink_kv : nullptr; p.nsink = nsink > 0 ? nsink : 0;
  p.gate = gate; p.gate_mode = (int)gm; p.sm_scale = default_scale(sm_scale, DQK);
  p.B = B; p.S = S; p.T = T; p.H = H; p.DQK = DQK; p.DV = DV; p.q_off = T - S; p.out = out;
  return p;
}

static dsa_status sparse_attn_impl(dsa_dtype dtype, const void* q, const void* k, const void* v,
                                   const int32_t* idx, int K, const void* sink_k,
                                   const void* sink_v, int nsink, const void* gate,
                                   dsa_gate_mode gate_mode, float sm_scale, int B, int S, int T,
                                   int H, int DQK, int DV, dsa_attn_algo algo, void* out,
                                   void* ws, size_t ws_bytes, dsa_stream_t stream) {
  dsa_status st = dsa::check_attn_common(dtype, q, k, v, gate, gate_mode, sm_scale, B, S, T, H,
                                         H, DQK, DV, out);
  if (st != DSA_OK) return st;
  if ((st = dsa::check_idx_args(idx, K)) != DSA_OK) return st;
  REQUIRE(algo >= DSA_ATTN_AUTO && algo <= DSA_ATTN_MASKED_TILE, DSA_ERR_INVALID_ARG,
          "unknown attention algorithm %d", (int)algo);
  if ((st = check_sinks(sink_k, sink_v, nsink)) != DSA_OK) return st;
  const int alg = choose_algo(algo, dtype, B, S, T, H, DQK, DV, K);
  REQUIRE(alg != kNone, DSA_ERR_UNSUPPORTED,
          "the masked-tile algorithm needs bf16, DQK in {128,192} and DV == 128");
  const size_t need =
      dsa_sparse_attn_sinks_workspace_bytes(dtype, B, S, T, H, DQK, DV, K, nsink, algo);
  REQUIRE(ws_bytes >= need && (need == 0 || ws != nullptr), DSA_ERR_INVALID_ARG,
          "workspace too small: %zu bytes given, %zu needed", ws_bytes, need);
  REQUIRE(ws == nullptr || aligned16(ws), DSA_ERR_UNSUPPORTED, "workspace must be 16-byte aligned");
  dsa::AttnProblem p{};
  p.dtype = (int)dtype; p.q = q; p.k = k; p.v = v; p.idx = idx; p.K = K; p.window = 0;
  p.gate = gate; p.gate_mode = (int)gate_mode; p.sm_scale = default_scale(sm_scale, DQK);
  p.B = B; p.S = S; p.T = T; p.H = H; p.HKV = H; p.DQK = DQK; p.DV = DV; p.q_off = T - S;
  p.out = out;
  p.sink_k = nsink > 0 ? sink_k : nullptr; p.sink_v = nsink > 0 ? sink_v : nullptr;
  p.nsink = nsink;
  cudaStream_t s = (cudaStream_t)stream;
  if (alg == kMasked) {
    uint32_t* mask = static_cast<uint32_t*>(ws);
    const int stride = dsa::mask_stride_words(T);
    st = cuda_status(dsa::launch_idx_to_mask(idx, B, S, T, K, T - S, mask, stride, s),
                     "dsa_sparse_attn/mask");
    if (st != DSA_OK) return st;
    return cuda_status(dsa::launch_masked_attn(p, mask, stride,
                                               dsa::masked_attn_blocks(mask, B, S, T), s),
                       "dsa_sparse_attn");
  }
  return cuda_status(dsa::launch_gather_attn(p, ws, ws_bytes, s), "dsa_sparse_attn");
}

dsa_status dsa_sparse_attn(dsa_dtype dtype, const void* q, const void* k, const void* v,
                           const int32_t* idx, int K, const void* gate,
                           dsa_gate_mode gate_mode, float sm_scale, int B, int S, int T,
                           int H, int DQK, int DV, dsa_attn_algo algo, void* out, void* ws,
                           size_t ws_bytes, dsa_stream_t stream) {
  return sparse_attn_impl(dtype, q, k, v, idx, K, nullptr, nullptr, 0, gate, gate_mode, sm_scale,
                          B, S, T, H, DQK, DV, algo, out, ws, ws_bytes, stream);
}

dsa_status dsa_sparse_attn_sinks(dsa_dtype dtype, const void* q, const void* k, const void* v,
                                 const int32_t* idx, int K, const void* sink_k,
                                 const void* sink_v, int nsink, const void* gate,
                                 dsa_gate_mode gate_mode, float sm_scale, int B, int S, int T,
                                 int H, int DQK, int DV, dsa_attn_algo algo, void* out, void* ws,
                                 size_t ws_bytes, dsa_stream_t stream) {
  REQUIRE(nsink > 0, DSA_ERR_INVALID_ARG, "nsink must be positive (use dsa_sparse_attn)");
  return sparse_attn_impl(dtype, q, k, v, idx, K, sink_k, sink_v, nsink, gate, gate_mode,
                          sm_scale, B, S, T, H, DQK, DV, algo, out, ws, ws_bytes, stream);
}

size_t dsa_sparse_attn_latent_workspace_bytes(int B, int S, int H, int K, int nsink) {
  if (B <= 0 || S <= 0 || H <= 0 || K <= 0 || nsink < 0) return 0;
  return dsa::latent_attn_workspace_bytes(B, S, H, K, nsink);
}

dsa_status dsa_sparse_attn_latent(dsa_dtype dtype, const void* q, const void* kv,
                                  const int32_t* idx, int K, const void* sink_kv, int nsink,
                                  const void* gate, dsa_gate_mode gate_mode, float sm_scale,
                                  int B, int S, int T, int H, int DQK, int DV, void* out,
                                  void* ws, size_t ws_bytes, dsa_stream_t stream) {
  dsa_status st = check_latent(dtype, q, kv, sink_kv, nsink, gate, gate_mode, sm_scale, B, S, T,
                               H, DQK, DV, out);
  if (st != DSA_OK) return st;
  REQUIRE(idx != nullptr && K > 0, DSA_ERR_INVALID_ARG, "idx must be given with K > 0");
  REQUIRE(aligned16(idx), DSA_ERR_UNSUPPORTED, "idx must be 16-byte aligned");
  const size_t need = dsa_sparse_attn_latent_workspace_bytes(B, S, H, K, nsink);
  REQUIRE(ws_bytes >= need && (need == 0 || ws != nullptr), DSA_ERR_INVALID_ARG,
          "workspace too small: %zu bytes given, %zu needed", ws_bytes, need);
  REQUIRE(ws == nullptr || aligned16(ws), DSA_ERR_UNSUPPORTED, "workspace must be 16-byte aligned");
  const dsa::LatentProblem p = latent_problem(q, kv, idx, K, sink_kv, nsink, gate, gate_mode,
                                              sm_scale, B, S, T, H, DQK, DV, out);
  return cuda_status(dsa::launch_latent_attn(p, ws, ws_bytes, (cudaStream_t)stream),
                     "dsa_sparse_attn_latent");
}

static dsa_status window_attn_impl(dsa_dtype dtype, const void* q, const void* k, const void* v,
                                   const void* sink_k, const void* sink_v, int nsink,
                                   const void* gate, dsa_gate_mode gate_mode, float sm_scale,
                                   int window, int B, int S, int T, int H, int HKV, int DQK,
                                   int DV, dsa_attn_algo algo, void* out, dsa_stream_t stream) {
  dsa_status st = dsa::check_attn_common(dtype, q, k, v, gate, gate_mode, sm_scale, B, S, T, H, HKV,
                                    DQK, DV, out);
  if (st != DSA_OK) return st;
  REQUIRE(window > 0, DSA_ERR_INVALID_ARG, "window must be positive");
  if ((st = check_sinks(sink_k, sink_v, nsink)) != DSA_OK) return st;
  REQUIRE(algo >= DSA_ATTN_AUTO && algo <= DSA_ATTN_MASKED_TILE, DSA_ERR_INVALID_ARG,
          "unknown attention algorithm %d", (int)algo);
  const bool tc = dsa::masked_attn_supported((int)dtype, DQK, DV);
  REQUIRE(algo != DSA_ATTN_MASKED_TILE || tc, DSA_ERR_UNSUPPORTED,
          "the masked-tile algorithm needs bf16, DQK in {128,192} and DV == 128");
  dsa::AttnProblem p{};
  p.dtype = (int)dtype; p.q = q; p.k = k; p.v = v; p.idx = nullptr; p.K = 0; p.window = window;
  p.gate = gate; p.gate_mode = (int)gate_mode; p.sm_scale = default_scale(sm_scale, DQK);
  p.B = B; p.S = S; p.T = T; p.H = H; p.HKV = HKV; p.DQK = DQK; p.DV = DV; p.q_off = T - S;
  p.out = out;
  p.sink_k = nsink > 0 ? sink_k : nullptr; p.sink_v = nsink > 0 ? sink_v : nullptr;
  p.nsink = nsink;
  cudaStream_t s = (cudaStream_t)stream;
  // the band is dense work for every query block with at least a few rows: tensor cores
  if (algo == DSA_ATTN_MASKED_TILE || (algo == DSA_ATTN_AUTO && tc && S >= 64))
    return cuda_status(dsa::launch_masked_attn(p, nullptr, 0, nullptr, s), "dsa_window_attn");
  return cuda_status(dsa::launch_gather_attn(p, nullptr, 0, s), "dsa_window_attn");
}

dsa_status dsa_window_attn(dsa_dtype dtype, const void* q, const void* k, const void* v,
                           const void* gate, dsa_gate_mode gate_mode, float sm_scale,
                           int window, int B, int S, int T, int H, int HKV, int DQK, int DV,
                           dsa_attn_algo algo, void* out, dsa_stream_t stream) {
  return window_attn_impl(dtype, q, k, v, nullptr, nullptr, 0, gate, gate_mode, sm_scale, window,
                          B, S, T, H, HKV, DQK, DV, algo, out, stream);
}

dsa_status dsa_window_attn_sinks(dsa_dtype dtype, const void* q, const void* k, const void* v,
                                 const void* sink_k, const void* sink_v, int nsink,
                                 const void* gate, dsa_gate_mode gate_mode, float sm_scale,
                                 int window, int B, int S, int T, int H, int HKV, int DQK,
                                 int DV, dsa_attn_algo algo, void* out, dsa_stream_t stream) {
  REQUIRE(nsink > 0, DSA_ERR_INVALID_ARG, "nsink must be positive (use dsa_window_attn)");
  return window_attn_impl(dtype, q, k, v, sink_k, sink_v, nsink, gate, gate_mode, sm_scale,
                          window, B, S, T, H, HKV, DQK, DV, algo, out, stream);
}

// ----------------------------------------------------------------------------- forward
// The element type of q_idx / k_idx: the attention dtype, or e4m3 when asked for.
static dsa_dtype index_dtype(const dsa_forward_args* a) {
  return a->index_dtype == DSA_INDEX_E4M3 ? DSA_E4M3 : a->dtype;
}

static dsa_status check_forward(const dsa_forward_args* a) {
  REQUIRE(a != nullptr, DSA_ERR_INVALID_ARG, "null args");
  REQUIRE(a->index_dtype == DSA_INDEX_AS_DTYPE || a->index_dtype == DSA_INDEX_E4M3,
          DSA_ERR_INVALID_ARG, "unknown index dtype %d", (int)a->index_dtype);
  REQUIRE(a->dtype != DSA_E4M3, DSA_ERR_INVALID_ARG,
          "e4m3 is an indexer input type (index_dtype), not an attention dtype");
  REQUIRE(a->index_dtype != DSA_INDEX_E4M3 || a->indexer == DSA_INDEXER_PER_HEAD,
          DSA_ERR_UNSUPPORTED, "the collapsed indexer takes bf16 inputs");
  dsa_status st = check_index_args(index_dtype(a), a->q_idx, a->k_idx, a->w, a->index_scale,
                                   a->relu,
                                   a->B, a->S, a->T, a->HI, a->DI,
                                   a->scores_out ? (const void*)a->scores_out : (const void*)a);
  if (st != DSA_OK) return st;
  REQUIRE(a->attn_form == DSA_ATTN_EXPANDED || a->attn_form == DSA_ATTN_LATENT,
          DSA_ERR_INVALID_ARG, "unknown attention form %d", (int)a->attn_form);
  const bool latent = a->attn_form == DSA_ATTN_LATENT;
  st = latent ? check_latent(a->dtype, a->q, a->k, a->sink_k, a->nsink, a->gate, a->gate_mode,
                             a->sm_scale, a->B, a->S, a->T, a->H, a->DQK, a->DV, a->out)
              : dsa::check_attn_common(a->dtype, a->q, a->k, a->v, a->gate, a->gate_mode,
                                  a->sm_scale, a->B, a->S, a->T, a->H, a->H, a->DQK, a->DV,
                                  a->out);
  if (st != DSA_OK) return st;
  REQUIRE(a->K > 0, DSA_ERR_INVALID_ARG, "K must be positive");
  REQUIRE(a->attn_algo >= DSA_ATTN_AUTO && a->attn_algo <= DSA_ATTN_MASKED_TILE,
          DSA_ERR_INVALID_ARG, "unknown attention algorithm %d", (int)a->attn_algo);
  REQUIRE(a->idx_out == nullptr || aligned16(a->idx_out), DSA_ERR_UNSUPPORTED,
          "idx_out must be 16-byte aligned");
  REQUIRE(a->indexer == DSA_INDEXER_PER_HEAD || a->indexer == DSA_INDEXER_COLLAPSED ||
              a->indexer == DSA_INDEXER_FUSED,
          DSA_ERR_INVALID_ARG, "unknown indexer mode %d", (int)a->indexer);
  if (a->indexer == DSA_INDEXER_FUSED) {
    const int k_eff = a->K < a->T ? a->K : a->T;
    REQUIRE(a->index_dtype == DSA_INDEX_AS_DTYPE &&
                fused_supported(a->dtype, a->HI, a->DI, a->T, k_eff),
            DSA_ERR_UNSUPPORTED,
            "the fused indexer needs bf16 inputs, HI in {16,32}, DI in {64,128} and T, K small "
            "enough for the candidate select");
    REQUIRE(a->topk_fallback_out == nullptr || aligned16(a->topk_fallback_out),
            DSA_ERR_UNSUPPORTED, "topk_fallback_out must be 16-byte aligned");
  }
  if (!latent && (st = check_sinks(a->sink_k, a->sink_v, a->nsink)) != DSA_OK) return st;
  if (a->indexer == DSA_INDEXER_COLLAPSED) return check_collapsed(a->dtype, a->relu, a->DI);
  return DSA_OK;
}

struct FwdLayout {
  size_t idx_off, attn_off, mask_off, qc_off, scores_off, total_full, total_min;
  size_t fused_off;  // DSA_INDEXER_FUSED: its workspace (fused_layout) starts here
  int k_eff, alg, mask_stride;
};

static FwdLayout forward_layout(const dsa_forward_args* a) {
  FwdLayout L{};
  L.k_eff = a->K < a->T ? a->K : a->T;
  const bool latent = a->attn_form == DSA_ATTN_LATENT;
  L.alg = latent ? kLatent
                 : choose_algo(a->attn_algo, a->dtype, a->B, a->S, a->T, a->H, a->DQK, a->DV,
                               L.k_eff);
  L.mask_stride = dsa::mask_stride_words(a->T);
  size_t off = 0;
  L.idx_off = off;
  if (!a->idx_out) off += align256((size_t)a->B * a->S * L.k_eff * sizeof(int32_t));
  L.attn_off = off;
  if (latent)
    off += align256(dsa::latent_attn_workspace_bytes(a->B, a->S, a->H, L.k_eff,
                                                     a->nsink > 0 ? a->nsink : 0));
  else if (L.alg == kGather)
    off += align256(dsa::gather_attn_workspace_bytes(a->B, a->S, a->H, a->DV, L.k_eff,
                                                     a->nsink > 0 ? a->nsink : 0));
  L.mask_off = off;
  if (L.alg == kMasked) off += align256(mask_bytes(a->B, a->S, a->T));
  L.qc_off = off;
  if (a->indexer == DSA_INDEXER_COLLAPSED) off += align256(collapsed_q_bytes(a->B, a->S, a->DI));
  L.scores_off = off;
  L.fused_off = off;
  if (a->scores_out) {
    L.total_full = L.total_min = off;
  } else {
    L.total_full = off + align256((size_t)a->B * a->S * a->T * sizeof(float));
    L.total_min = off + align256((size_t)a->T * sizeof(float));
    if (a->indexer == DSA_INDEXER_FUSED)  // its layout ends with the full score matrix
      L.total_full = off + fused_layout(a->B, a->S, a->T, L.k_eff).total;
  }
  return L;
}

size_t dsa_forward_workspace_bytes(const dsa_forward_args* a) {
  if (!a || a->B <= 0 || a->S <= 0 || a->T <= 0 || a->K <= 0) return 0;
  return forward_layout(a).total_full;
}

size_t dsa_forward_min_workspace_bytes(const dsa_forward_args* a) {
  if (!a || a->B <= 0 || a->S <= 0 || a->T <= 0 || a->K <= 0) return 0;
  return forward_layout(a).total_min;
}

dsa_status dsa_forward(const dsa_forward_args* a, void* ws, size_t ws_bytes,
                       dsa_stream_t stream) {
  dsa_status st = check_forward(a);
  if (st != DSA_OK) return st;
  const FwdLayout L = forward_layout(a);
  REQUIRE(L.alg != kNone, DSA_ERR_UNSUPPORTED,
          "the masked-tile algorithm needs bf16, DQK in {128,192} and DV == 128");
  REQUIRE(ws_bytes >= L.total_min && (L.total_min == 0 || ws != nullptr), DSA_ERR_INVALID_ARG,
          "workspace too small: %zu bytes given, at least %zu needed", ws_bytes, L.total_min);
  REQUIRE(ws == nullptr || aligned16(ws), DSA_ERR_UNSUPPORTED, "workspace must be 16-byte aligned");
  cudaStream_t s = (cudaStream_t)stream;
  uint8_t* base = static_cast<uint8_t*>(ws);
  int32_t* idx = a->idx_out ? a->idx_out : reinterpret_cast<int32_t*>(base + L.idx_off);
  void* attn_ws = (base && (L.alg == kGather || L.alg == kLatent)) ? base + L.attn_off : nullptr;
  const bool collapsed = a->indexer == DSA_INDEXER_COLLAPSED;
  uint8_t* qc = collapsed ? base + L.qc_off : nullptr;
  const size_t attn_ws_bytes = L.mask_off - L.attn_off;
  uint32_t* mask = L.alg == kMasked ? reinterpret_cast<uint32_t*>(base + L.mask_off) : nullptr;
  const int B = a->B, S = a->S, T = a->T, q_off = T - S;
  const size_t es = esize(index_dtype(a));  // q_idx / k_idx elements
  const int write_masked = a->scores_out != nullptr;  // -inf only matters to the caller
  cudaEvent_t const* ev = reinterpret_cast<cudaEvent_t const*>(a->events);
  auto mark = [&](int i) -> dsa_status {
    return ev ? cuda_status(cudaEventRecord(ev[i], s), "dsa_forward/event") : DSA_OK;
  };
  if ((st = mark(0)) != DSA_OK) return st;
  // the fused indexer -> top-k needs its whole workspace and no score matrix output; else
  // the per-head path below computes the same indices
  const bool fused =
      a->indexer == DSA_INDEXER_FUSED && !a->scores_out && ws_bytes >= L.total_full;
  if (fused) {
    st = run_fused_index_topk(a->q_idx, a->k_idx, a->w, a->index_scale, a->relu, B, S, T,
                              a->HI, a->DI, L.k_eff, idx, mask, L.mask_stride,
                              base + L.fused_off, a->topk_fallback_out, s,
                              ev ? ev[1] : nullptr);
    if (st != DSA_OK || (st = mark(2)) != DSA_OK) return st;
  } else if (a->indexer == DSA_INDEXER_FUSED && a->topk_fallback_out &&
             (st = cuda_status(cudaMemsetAsync(a->topk_fallback_out, 0, sizeof(int32_t), s),
                               "dsa_forward/fallback flag")) != DSA_OK) {
    return st;
  }
  if (!fused && collapsed &&
      (st = run_collapse_q(a->q_idx, a->w, (long long)B * S, a->HI, a->DI, qc, s)) != DSA_OK)
    return st;

  if (fused) {
    // indices and the selection mask are done
  } else if (a->scores_out || ws_bytes >= L.total_full) {
    float* scores = a->scores_out ? a->scores_out : reinterpret_cast<float*>(base + L.scores_off);
    st = collapsed ? run_index_scores_collapsed(qc, a->k_idx, a->index_scale, a->relu, B, S, T,
                                                a->DI, q_off, scores, write_masked, s)
                   : run_index_scores(index_dtype(a), a->q_idx, a->k_idx, a->w,
                                      a->index_scale, a->relu, B, S, T, a->HI, a->DI, q_off,
                                      scores, write_masked, s);
    if (st != DSA_OK || (st = mark(1)) != DSA_OK) return st;
    st = cuda_status(dsa::launch_topk(scores, B, S, T, L.k_eff, q_off, idx, mask, L.mask_stride,
                                      s),
                     "dsa_forward/topk");
    if (st != DSA_OK || (st = mark(2)) != DSA_OK) return st;
  } else {
    // row blocks that fit the score buffer, one batch row at a time
    float* scores = reinterpret_cast<float*>(base + L.scores_off);
    const size_t avail = ws_bytes - L.scores_off;
    int rb = (int)(avail / ((size_t)T * sizeof(float)));
    if (rb > S) rb = S;
    for (int b = 0; b < B; ++b) {
      for (int s0 = 0; s0 < S; s0 += rb) {
        const int n = S - s0 < rb ? S - s0 : rb;
        const uint8_t* qi = static_cast<const uint8_t*>(a->q_idx) +
                            ((size_t)b * S + s0) * a->HI * a->DI * es;
        const uint8_t* ki = static_cast<const uint8_t*>(a->k_idx) + (size_t)b * T * a->DI * es;
        const float* wb = a->w + ((size_t)b * S + s0) * a->HI;
        // this block's first query sits at key position q_off + s0
        const uint8_t* qcb = collapsed ? qc + ((size_t)b * S + s0) * 2 * a->DI * 2 : nullptr;
        st = collapsed ? run_index_scores_collapsed(qcb, ki, a->index_scale, a->relu, 1, n, T,
                                                    a->DI, q_off + s0, scores, 0, s)
                       : run_index_scores(index_dtype(a), qi, ki, wb, a->index_scale, a->relu,
                                          1, n, T, a->HI, a->DI, q_off + s0, scores, 0, s);
        if (st != DSA_OK) return st;
        const size_t row0 = (size_t)b * S + s0;
        st = cuda_status(dsa::launch_topk(scores, 1, n, T, L.k_eff, q_off + s0,
                                          idx + row0 * L.k_eff,
                                          mask ? mask + row0 * L.mask_stride : nullptr,
                                          L.mask_stride, s),
                         "dsa_forward/topk");
        if (st != DSA_OK) return st;
      }
    }
    // row blocks interleave the two stages: both boundary events mark their end
    if ((st = mark(1)) != DSA_OK || (st = mark(2)) != DSA_OK) return st;
  }
  if (L.alg == kLatent) {
    const dsa::LatentProblem lp =
        latent_problem(a->q, a->k, idx, L.k_eff, a->sink_k, a->nsink, a->gate, a->gate_mode,
                       a->sm_scale, B, S, T, a->H, a->DQK, a->DV, a->out);
    st = cuda_status(dsa::launch_latent_attn(lp, attn_ws, attn_ws_bytes, s), "dsa_forward/attn");
    if (st != DSA_OK) return st;
    return mark(3);
  }
  dsa::AttnProblem p{};
  p.dtype = (int)a->dtype; p.q = a->q; p.k = a->k; p.v = a->v; p.idx = idx; p.K = L.k_eff;
  p.window = 0; p.gate = a->gate; p.gate_mode = (int)a->gate_mode;
  p.sm_scale = default_scale(a->sm_scale, a->DQK);
  p.B = B; p.S = S; p.T = T; p.H = a->H; p.HKV = a->H; p.DQK = a->DQK; p.DV = a->DV;
  p.q_off = q_off; p.out = a->out;
  if (a->nsink > 0) {
    p.sink_k = a->sink_k; p.sink_v = a->sink_v; p.nsink = a->nsink;
  }
  if (L.alg == kMasked)
    st = cuda_status(dsa::launch_masked_attn(p, mask, L.mask_stride,
                                             dsa::masked_attn_blocks(mask, B, S, T), s),
                     "dsa_forward/attn");
  else
    st = cuda_status(dsa::launch_gather_attn(p, attn_ws, attn_ws_bytes, s), "dsa_forward/attn");
  if (st != DSA_OK) return st;
  return mark(3);
}

}  // extern "C"
