// dspark_draft_sample_static: the draft-sampling entry point for callers that
// cannot allocate device memory.
//
// dspark_draft_sample needs a caller-owned workspace for its per-chunk softmax
// partials. Some callers have no way to provide one: code that runs inside
// another runtime's memory manager (an inference server or framework whose
// caching allocator has already reserved the device memory, so an extra
// cudaMalloc can fail or corrupt the pool's accounting), plug-in hosts that
// hand a kernel only its input and output buffers, and latency-critical paths
// where cudaMalloc's implicit device synchronisation is not acceptable. This
// variant keeps that scratch in a fixed array that lives in the library's own
// device image instead.
//
// The array is a file-scope __device__ object of kStaticScratchBytes (8 MiB):
// every GPU on which the library is loaded holds it until the process exits.
// In host code its name is only a host-side stand-in, so its device address is
// looked up with cudaGetSymbolAddress, once per device, on the first call made
// while that device is current; that first call should therefore come before
// any stream capture. No call allocates or frees memory.
#include <climits>
#include <mutex>

#include "common.cuh"
#include "draft.cuh"
#include "draft_tc.cuh"

namespace dspark {
namespace {

constexpr size_t kStaticScratchBytes = size_t(8) << 20;
constexpr int kMaxDevices = 64;

// status block (first 256 bytes) followed by the chunk partials
__device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices];  // device address of g_static_scratch, per device

int scratch_for_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DSPARK_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return DSPARK_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr)
      return DSPARK_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return DSPARK_OK;
}

// {status bits, lowest offending request or -1} into the caller's buffer
__global__ void copy_status(const Status* st, int32_t* out) {
  out[0] = (int32_t)st->code;
  out[1] = st->first_bad_enc ? INT_MAX - st->first_bad_enc : -1;
}

}  // namespace
}  // namespace dspark

using namespace dspark;

extern "C" int dspark_draft_sample_static(const void* base, const void* U, const void* W,
                                          const float* bias_scale, const int32_t* last_tok,
                                          const float* temp, int B, int K, int V, int r, int dtype,
                                          uint64_t seed, uint64_t round_id, int32_t* x, void* d,
                                          float* q_lse, float* q_tok, int32_t* status_out,
                                          dspark_stream_t stream) {
  if (!base || !U || !W || !last_tok || !temp || !x || !d || !q_lse || !q_tok)
    return DSPARK_ERR_INVALID_ARG;
  if (dtype != DSPARK_F32 && dtype != DSPARK_BF16) return DSPARK_ERR_INVALID_ARG;
  if (B < 1 || B > 65535 || K < 1 || K > 64 || V < 8 || V >= (1 << 24) || V % 8 != 0 || r < 1 ||
      r > 1024)
    return DSPARK_ERR_INVALID_ARG;
  if (dtype == DSPARK_BF16 && r % 16 != 0) return DSPARK_ERR_UNSUPPORTED;
  const uintptr_t mis = reinterpret_cast<uintptr_t>(base) | reinterpret_cast<uintptr_t>(U) |
                        reinterpret_cast<uintptr_t>(W) | reinterpret_cast<uintptr_t>(d);
  if (mis & 15u) return DSPARK_ERR_INVALID_ARG;
  const int nchunk = (V + kChunk - 1) / kChunk;
  if (kStatusBytes + (size_t)B * nchunk * sizeof(float2) > kStaticScratchBytes)
    return DSPARK_ERR_WORKSPACE;  // larger than the fixed scratch

  int dev = 0, major = 0, minor = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return DSPARK_ERR_CUDA;
  if (major != 10 || minor != 0) return DSPARK_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  if (int e = scratch_for_current_device(&scratch)) return e;

  cudaStream_t s = (cudaStream_t)stream;
  // the array keeps the previous call's contents: the status block must start at zero
  // (the partials are fully written before they are read)
  if (cudaMemsetAsync(scratch, 0, kStatusBytes, s) != cudaSuccess) return DSPARK_ERR_CUDA;

  DraftArgs a;
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
  a.q_norm = nullptr;
  a.status = static_cast<Status*>(scratch);
  a.R = nullptr;  // the Markov head
  a.H = nullptr;
  a.partials = reinterpret_cast<float2*>(static_cast<char*>(scratch) + kStatusBytes);
  a.nchunk = nchunk;
  // the launches of dspark_draft_sample: one cooperative launch for the whole
  // block where the tensor-core path applies (its grid-barrier counter lives
  // in the status block, which the scratch holds too), else two per position
  if (draft_round_tc_supported(a, sms)) {
    if (draft_round_tc_launch(a, sms, kDraftFreeSms, s) != cudaSuccess) return DSPARK_ERR_CUDA;
  } else {
    const bool tc = draft_tc_supported(a);
    for (int k = 1; k <= K; ++k) {
      cudaError_t e = tc ? draft_logits_tc_launch(a, k, sms, s) : draft_logits_simt_launch(a, k, s);
      if (e == cudaSuccess) e = draft_sample_launch(a, k, s);
      if (e != cudaSuccess) return DSPARK_ERR_CUDA;
    }
  }
  if (status_out) {
    copy_status<<<1, 1, 0, s>>>(a.status, status_out);
    if (cudaGetLastError() != cudaSuccess) return DSPARK_ERR_CUDA;
  }
  return DSPARK_OK;
}
