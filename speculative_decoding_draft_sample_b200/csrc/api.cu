// C ABI of libdspark.so: argument checks, workspace layout and launches.
// Declarations and the contract of every entry point are in include/dspark.h.
#include <climits>
#include <cstring>

#include "calib.cuh"
#include "common.cuh"
#include "draft.cuh"
#include "draft_tc.cuh"
#include "schedule.cuh"
#include "verify.cuh"

namespace dspark {
// defined in selftest.cu
cudaError_t selftest_waits_launch(Status* st, int32_t* result, cudaStream_t s);
}  // namespace dspark

using namespace dspark;

namespace {

constexpr int kAbiVersion = (3 << 16) | 2;

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

inline int nchunks(int V) { return (V + kChunk - 1) / kChunk; }

// Workspace layout shared by the calls of one round:
//   [status block 256][draft chunk partials][target-row statistics][work counter 256]
//   [verification order: B request indices]
// The statistics sit past the draft's partials, so that dspark_verify_target_stats
// may run on another stream while dspark_draft_sample runs (they share only the
// status block, which both update atomically).
inline size_t draft_region(int B, int V) { return round_up((size_t)B * nchunks(V) * sizeof(float2), 256); }
inline size_t stats_region(int B, int K, int V, int dtype) {
  return round_up((size_t)B * (K + 1) * stats_chunks(V, dtype) * sizeof(float2), 256);
}
inline size_t stats_offset(int B, int V) { return kStatusBytes + draft_region(B, V); }
inline size_t counter_offset(int B, int K, int V, int dtype) {
  return stats_offset(B, V) + stats_region(B, K, V, dtype);
}
inline size_t order_offset(int B, int K, int V, int dtype) { return counter_offset(B, K, V, dtype) + 256; }

bool shape_ok(int B, int K, int V, int dtype) {
  if (dtype != DSPARK_F32 && dtype != DSPARK_BF16) return false;
  if (B < 1 || B > 65535 || K < 1 || K > 64) return false;
  if (V < 8 || V >= (1 << 24) || V % 8 != 0) return false;
  return true;
}

// The fatbin carries sm_100a code only.
int device_check(int* num_sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DSPARK_ERR_CUDA;
  int major = 0, minor = 0, sms = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return DSPARK_ERR_CUDA;
  if (major != 10 || minor != 0) return DSPARK_ERR_UNSUPPORTED;
  if (num_sms) *num_sms = sms;
  return DSPARK_OK;
}

inline int cuda_status(cudaError_t e) { return e == cudaSuccess ? DSPARK_OK : DSPARK_ERR_CUDA; }

}  // namespace

extern "C" {

int dspark_version(void) { return kAbiVersion; }

int dspark_selftest_waits(int32_t* result, void* ws, size_t ws_bytes, dspark_stream_t stream) {
  if (!result || !ws || !aligned16(ws) || ws_bytes < kStatusBytes) return DSPARK_ERR_INVALID_ARG;
  int sms = 0;
  if (int e = device_check(&sms)) return e;
  return cuda_status(
      selftest_waits_launch(static_cast<Status*>(ws), result, (cudaStream_t)stream));
}

const char* dspark_status_string(int code) {
  switch (code) {
    case DSPARK_OK: return "ok";
    case DSPARK_ERR_INVALID_ARG: return "invalid argument (null pointer, size or alignment)";
    case DSPARK_ERR_UNSUPPORTED: return "unsupported dtype, shape or device";
    case DSPARK_ERR_CUDA: return "CUDA launch or runtime error";
    case DSPARK_ERR_WORKSPACE: return "workspace too small";
    case DSPARK_ERR_TIMEOUT: return "a bounded device wait gave up";
    default: return "unknown status";
  }
}

size_t dspark_workspace_bytes(int op, int B, int K, int V, int r, int dtype) {
  switch (op) {
    case DSPARK_OP_DRAFT:
      if (!shape_ok(B, K, V, dtype) || r < 1 || r > 1024) return 0;
      return kStatusBytes + draft_region(B, V);
    case DSPARK_OP_SCHEDULE:
      if (B < 1 || K < 1 || K > 64) return 0;
      return kStatusBytes;
    case DSPARK_OP_CALIB:
      if (B < 1 || K < 1 || K > 64) return 0;
      return calib_workspace_bytes(B, K);
    case DSPARK_OP_VERIFY:
      if (!shape_ok(B, K, V, dtype)) return 0;
      return order_offset(B, K, V, dtype) + round_up((size_t)B * sizeof(int32_t), 256);
    default:
      return 0;
  }
}

int dspark_clear_status(void* ws, dspark_stream_t stream) {
  if (!ws) return DSPARK_ERR_INVALID_ARG;
  return cuda_status(cudaMemsetAsync(ws, 0, kStatusBytes, (cudaStream_t)stream));
}

int dspark_read_status(void* ws, dspark_stream_t stream, uint32_t* code, int32_t* first_bad) {
  if (!ws) return DSPARK_ERR_INVALID_ARG;
  Status h;
  cudaError_t e = cudaMemcpyAsync(&h, ws, sizeof(h), cudaMemcpyDeviceToHost, (cudaStream_t)stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return DSPARK_ERR_CUDA;
  if (code) *code = h.code;
  if (first_bad) *first_bad = (h.first_bad_enc == 0) ? -1 : INT_MAX - h.first_bad_enc;
  return dspark_clear_status(ws, stream);
}

}  // extern "C"

namespace {

// Argument checks and DraftArgs of the draft entry points. `logits` / `pick`
// select which of the two kernels the caller is about to launch; the pointers
// only the other one reads may be null.
int draft_prepare(DraftArgs& a, int* sms, bool logits, bool pick, const void* base, const void* U,
                  const void* W, const float* bias_scale, const int32_t* last_tok, const float* temp,
                  int B, int K, int V, int r, int dtype, uint64_t seed, uint64_t round_id, int32_t* x,
                  void* d, float* q_lse, float* q_tok, float* q_norm, void* ws, size_t ws_bytes) {
  if (!last_tok || !temp || !x || !d || !ws) return DSPARK_ERR_INVALID_ARG;
  if (logits && (!base || !U || !W)) return DSPARK_ERR_INVALID_ARG;
  if (pick && (!q_lse || !q_tok)) return DSPARK_ERR_INVALID_ARG;
  if (!shape_ok(B, K, V, dtype) || r < 1 || r > 1024) return DSPARK_ERR_INVALID_ARG;
  if (logits && dtype == DSPARK_BF16 && r % 16 != 0) return DSPARK_ERR_UNSUPPORTED;
  if (!aligned16(d) || !aligned16(ws)) return DSPARK_ERR_INVALID_ARG;
  if (logits && (!aligned16(base) || !aligned16(U) || !aligned16(W))) return DSPARK_ERR_INVALID_ARG;
  if (ws_bytes < dspark_workspace_bytes(DSPARK_OP_DRAFT, B, K, V, r, dtype))
    return DSPARK_ERR_WORKSPACE;
  if (int e = device_check(sms)) return e;
  a.base = base;
  a.U = U;
  a.W = W;
  a.bias_scale = bias_scale;
  a.last_tok = last_tok;
  a.temp = temp;
  a.B = B;
  a.K = K;
  a.V = V;
  a.r = r;
  a.dtype = dtype;
  a.seed = seed;
  a.round_id = round_id;
  a.x = x;
  a.d = d;
  a.q_lse = q_lse;
  a.q_tok = q_tok;
  a.q_norm = reinterpret_cast<float2*>(q_norm);
  a.status = static_cast<Status*>(ws);
  a.partials = reinterpret_cast<float2*>(static_cast<char*>(ws) + kStatusBytes);
  a.nchunk = nchunks(V);
  a.R = nullptr;  // the Markov head unless the caller adds the recurrent one
  a.H = nullptr;
  return DSPARK_OK;
}

cudaError_t launch_logits(const DraftArgs& a, int k, int sms, cudaStream_t s) {
  return draft_tc_supported(a) ? draft_logits_tc_launch(a, k, sms, s) : draft_logits_simt_launch(a, k, s);
}

// All K positions: one cooperative launch for the whole block when the
// tensor-core path applies and every M-tile gets its own CTAs (free_sms SMs
// left to other streams); otherwise two launches per position (the same
// kernels, so the results are identical).
int draft_run(const DraftArgs& a, int sms, int free_sms, cudaStream_t s) {
  if (draft_round_tc_supported(a, sms)) return cuda_status(draft_round_tc_launch(a, sms, free_sms, s));
  for (int k = 1; k <= a.K; ++k) {
    cudaError_t e = launch_logits(a, k, sms, s);
    if (e == cudaSuccess) e = draft_sample_launch(a, k, s);
    if (e != cudaSuccess) return DSPARK_ERR_CUDA;
  }
  return DSPARK_OK;
}

}  // namespace

extern "C" {

int dspark_draft_sample(const void* base, const void* U, const void* W, const float* bias_scale,
                        const int32_t* last_tok, const float* temp, int B, int K, int V, int r,
                        int dtype, uint64_t seed, uint64_t round_id, int32_t* x, void* d,
                        float* q_lse, float* q_tok, float* q_norm, void* ws, size_t ws_bytes,
                        dspark_stream_t stream) {
  DraftArgs a;
  int sms = 0;
  if (int e = draft_prepare(a, &sms, true, true, base, U, W, bias_scale, last_tok, temp, B, K, V, r,
                            dtype, seed, round_id, x, d, q_lse, q_tok, q_norm, ws, ws_bytes))
    return e;
  return draft_run(a, sms, kDraftFreeSms, (cudaStream_t)stream);
}

int dspark_draft_sample_recurrent(const void* base, const void* U, const void* W, const void* R,
                                  const float* bias_scale, const int32_t* last_tok,
                                  const float* temp, int B, int K, int V, int r, int dtype,
                                  uint64_t seed, uint64_t round_id, int32_t* x, void* d,
                                  float* q_lse, float* q_tok, float* q_norm, void* h, void* ws,
                                  size_t ws_bytes, dspark_stream_t stream) {
  if (!R || !h) return DSPARK_ERR_INVALID_ARG;
  if (!aligned16(R) || !aligned16(h) || r % 8 != 0) return DSPARK_ERR_INVALID_ARG;
  DraftArgs a;
  int sms = 0;
  if (int e = draft_prepare(a, &sms, true, true, base, U, W, bias_scale, last_tok, temp, B, K, V, r,
                            dtype, seed, round_id, x, d, q_lse, q_tok, q_norm, ws, ws_bytes))
    return e;
  a.R = R;
  a.H = h;
  // the same launches as dspark_draft_sample; the draw of every position also
  // forms the next position's state, and the bias rows come from the states
  return draft_run(a, sms, kDraftFreeSms, (cudaStream_t)stream);
}

int dspark_draft_sample_beside(const void* base, const void* U, const void* W, const void* R,
                               const float* bias_scale, const int32_t* last_tok, const float* temp,
                               int B, int K, int V, int r, int dtype, uint64_t seed,
                               uint64_t round_id, int32_t* x, void* d, float* q_lse, float* q_tok,
                               float* q_norm, void* h, int free_sms, void* ws, size_t ws_bytes,
                               dspark_stream_t stream) {
  if (free_sms < 0) return DSPARK_ERR_INVALID_ARG;
  if (R && (!h || !aligned16(R) || !aligned16(h) || r % 8 != 0)) return DSPARK_ERR_INVALID_ARG;
  DraftArgs a;
  int sms = 0;
  if (int e = draft_prepare(a, &sms, true, true, base, U, W, bias_scale, last_tok, temp, B, K, V, r,
                            dtype, seed, round_id, x, d, q_lse, q_tok, q_norm, ws, ws_bytes))
    return e;
  if (R) {
    a.R = R;
    a.H = h;
  }
  return draft_run(a, sms, free_sms, (cudaStream_t)stream);
}

int dspark_draft_logits(const void* base, const void* U, const void* W, const float* bias_scale,
                        const int32_t* last_tok, const int32_t* x, const float* temp, int B, int K,
                        int V, int r, int dtype, int k, void* d, void* ws, size_t ws_bytes,
                        dspark_stream_t stream) {
  if (k < 1 || k > K) return DSPARK_ERR_INVALID_ARG;
  DraftArgs a;
  int sms = 0;
  if (int e = draft_prepare(a, &sms, true, false, base, U, W, bias_scale, last_tok, temp, B, K, V, r,
                            dtype, 0, 0, const_cast<int32_t*>(x), d, nullptr, nullptr, nullptr, ws,
                            ws_bytes))
    return e;
  return cuda_status(launch_logits(a, k, sms, (cudaStream_t)stream));
}

int dspark_draft_pick(const void* d, const int32_t* last_tok, const float* temp, int B, int K, int V,
                      int dtype, uint64_t seed, uint64_t round_id, int k, int32_t* x, float* q_lse,
                      float* q_tok, float* q_norm, void* ws, size_t ws_bytes, dspark_stream_t stream) {
  if (k < 1 || k > K) return DSPARK_ERR_INVALID_ARG;
  DraftArgs a;
  if (int e = draft_prepare(a, nullptr, false, true, nullptr, nullptr, nullptr, nullptr, last_tok, temp,
                            B, K, V, 16, dtype, seed, round_id, x, const_cast<void*>(d), q_lse, q_tok,
                            q_norm, ws, ws_bytes))
    return e;
  return cuda_status(draft_sample_launch(a, k, (cudaStream_t)stream));
}

int dspark_prefix_schedule(const float* conf_logit, const float* pos_temp, const float* step_cost,
                           float fixed_cost, int B, int K, int mode, float threshold, int32_t* cut,
                           float* survival, void* ws, size_t ws_bytes, dspark_stream_t stream) {
  if (!conf_logit || !pos_temp || !cut || !survival || !ws) return DSPARK_ERR_INVALID_ARG;
  if (mode != DSPARK_CUT_COST && mode != DSPARK_CUT_THRESHOLD && mode != DSPARK_CUT_NONE)
    return DSPARK_ERR_INVALID_ARG;
  if (mode == DSPARK_CUT_COST && !step_cost) return DSPARK_ERR_INVALID_ARG;
  if (B < 1 || K < 1 || K > 64) return DSPARK_ERR_INVALID_ARG;
  if (mode == DSPARK_CUT_COST && ((long long)B * K > kMaxScheduleItems || B > kMaxScheduleItems))
    return DSPARK_ERR_UNSUPPORTED;
  if (!aligned16(ws)) return DSPARK_ERR_INVALID_ARG;
  if (ws_bytes < dspark_workspace_bytes(DSPARK_OP_SCHEDULE, B, K, 8, 1, DSPARK_F32))
    return DSPARK_ERR_WORKSPACE;
  if (int e = device_check(nullptr)) return e;
  SchedArgs a;
  a.conf_logit = conf_logit;
  a.pos_temp = pos_temp;
  a.step_cost = step_cost;
  a.fixed_cost = fixed_cost;
  a.B = B;
  a.K = K;
  a.mode = mode;
  a.threshold = threshold;
  a.cut = cut;
  a.survival = survival;
  a.status = static_cast<Status*>(ws);
  return cuda_status(prefix_schedule_launch(a, (cudaStream_t)stream));
}

}  // extern "C"

namespace {

int stats_prepare(StatsArgs& sa, int* sms, const void* target, const int32_t* cut, const float* temp,
                  int B, int K, int V, int dtype, void* ws, size_t ws_bytes) {
  if (!target || !temp || !ws) return DSPARK_ERR_INVALID_ARG;
  if (!shape_ok(B, K, V, dtype)) return DSPARK_ERR_INVALID_ARG;
  if (!aligned16(target) || !aligned16(ws)) return DSPARK_ERR_INVALID_ARG;
  if (ws_bytes < dspark_workspace_bytes(DSPARK_OP_VERIFY, B, K, V, 1, dtype)) return DSPARK_ERR_WORKSPACE;
  if (int e = device_check(sms)) return e;
  char* w = static_cast<char*>(ws);
  sa.target = target;
  sa.cut = cut;
  sa.temp = temp;
  sa.B = B;
  sa.K = K;
  sa.V = V;
  sa.dtype = dtype;
  sa.partials = reinterpret_cast<float2*>(w + stats_offset(B, V));
  sa.nchunk = stats_chunks(V, dtype);
  sa.next = reinterpret_cast<unsigned long long*>(w + counter_offset(B, K, V, dtype));
  sa.order = reinterpret_cast<int32_t*>(w + order_offset(B, K, V, dtype));
  sa.status = static_cast<Status*>(ws);
  return DSPARK_OK;
}

int verify_decide(const void* target, const void* d, const int32_t* x, const float* q_tok,
                  const float* q_norm, const int32_t* cut, const float* temp, int B, int K, int V,
                  int dtype, uint64_t seed, uint64_t round_id, int32_t* accepted, int32_t* out,
                  int32_t* n_emit, void* ws, size_t ws_bytes, cudaStream_t s, bool with_stats) {
  if (!target || !d || !x || !q_tok || !temp || !accepted || !out || !n_emit || !ws)
    return DSPARK_ERR_INVALID_ARG;
  if (!aligned16(d)) return DSPARK_ERR_INVALID_ARG;
  StatsArgs sa;
  int sms = 0;
  if (int e = stats_prepare(sa, &sms, target, cut, temp, B, K, V, dtype, ws, ws_bytes)) return e;
  if (with_stats) {
    cudaError_t e = target_stats_launch(sa, sms, s);
    if (e != cudaSuccess) return DSPARK_ERR_CUDA;
  }
  VerifyArgs a;
  a.target = target;
  a.d = d;
  a.x = x;
  a.q_tok = q_tok;
  a.q_norm = reinterpret_cast<const float2*>(q_norm);
  a.cut = cut;
  a.temp = temp;
  a.B = B;
  a.K = K;
  a.V = V;
  a.dtype = dtype;
  a.seed = seed;
  a.round_id = round_id;
  a.accepted = accepted;
  a.out = out;
  a.n_emit = n_emit;
  a.status = static_cast<Status*>(ws);
  a.stats = sa.partials;
  a.nstat = sa.nchunk;
  a.order = cut ? sa.order : nullptr;  // written by the statistics pass
  const int C = verify_cluster_size(B, V, dtype, sms);
  return cuda_status(verify_launch(a, C, s));
}

}  // namespace

extern "C" {

int dspark_verify_target_stats(const void* target, const int32_t* cut, const float* temp, int B,
                               int K, int V, int dtype, void* ws, size_t ws_bytes,
                               dspark_stream_t stream) {
  StatsArgs sa;
  int sms = 0;
  if (int e = stats_prepare(sa, &sms, target, cut, temp, B, K, V, dtype, ws, ws_bytes)) return e;
  return cuda_status(target_stats_launch(sa, sms, (cudaStream_t)stream));
}

int dspark_verify_from_stats(const void* target, const void* d, const int32_t* x,
                             const float* q_tok, const float* q_norm, const int32_t* cut,
                             const float* temp, int B, int K, int V, int dtype, uint64_t seed,
                             uint64_t round_id, int32_t* accepted, int32_t* out, int32_t* n_emit,
                             void* ws, size_t ws_bytes, dspark_stream_t stream) {
  return verify_decide(target, d, x, q_tok, q_norm, cut, temp, B, K, V, dtype, seed, round_id,
                       accepted, out, n_emit, ws, ws_bytes, (cudaStream_t)stream, false);
}

int dspark_verify(const void* target, const void* d, const int32_t* x, const float* q_tok,
                  const float* q_norm,
                  const int32_t* cut, const float* temp, int B, int K, int V, int dtype,
                  uint64_t seed, uint64_t round_id, int32_t* accepted, int32_t* out,
                  int32_t* n_emit, void* ws, size_t ws_bytes, dspark_stream_t stream) {
  return verify_decide(target, d, x, q_tok, q_norm, cut, temp, B, K, V, dtype, seed, round_id,
                       accepted, out, n_emit, ws, ws_bytes, (cudaStream_t)stream, true);
}

int dspark_sts_fit(const float* conf_logit, const uint8_t* survived, int N, int K, float* T_out,
                   int32_t* index_out, float* ece_before, float* ece_after, void* ws,
                   size_t ws_bytes, dspark_stream_t stream) {
  if (!conf_logit || !survived || !T_out || !ws) return DSPARK_ERR_INVALID_ARG;
  if (N < 1 || K < 1 || K > 64) return DSPARK_ERR_INVALID_ARG;
  if (!aligned16(ws)) return DSPARK_ERR_INVALID_ARG;
  if (ws_bytes < dspark_workspace_bytes(DSPARK_OP_CALIB, N, K, 8, 1, DSPARK_F32))
    return DSPARK_ERR_WORKSPACE;
  if (int e = device_check(nullptr)) return e;
  CalibArgs a;
  a.z = conf_logit;
  a.y = survived;
  a.N = N;
  a.K = K;
  a.T = T_out;
  a.index = index_out;
  return cuda_status(calib_launch(a, ws, ece_before, ece_after, (cudaStream_t)stream));
}

}  // extern "C"
