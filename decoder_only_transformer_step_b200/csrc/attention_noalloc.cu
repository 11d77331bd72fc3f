// Attention backward for callers that cannot allocate device memory.
//
// gpt2_op_attention_bwd_bf16 needs fp32 scratch (the dQ accumulator and the
// per-row D = rowsum(dO * O) vector) that the caller passes in.  Some callers
// have no way to provide it: a host that hands a plug-in only its input and
// output buffers, or a runtime that has already reserved the device memory for
// its own caching allocator, where a raw cudaMalloc fails or would fight that
// allocator; cudaMalloc also synchronises the device, which latency-sensitive
// loops avoid.  This entry point keeps its scratch in a fixed-size array
// compiled into the library instead, so it allocates nothing.
//
// Cost of that choice: the array occupies kScratchFloats * 4 bytes (16 MiB) on
// every GPU that loads the library, until the process exits; problems whose
// scratch need is larger are rejected; and all calls share the one array, so
// calls that overlap on the GPU (different streams, no ordering) race on it.
#include <atomic>

#include "common.cuh"
#include "internal.h"

// dQ accumulator (B*T*H*hd floats) followed by D (B*H*T floats).
static constexpr size_t kScratchFloats = size_t(4) << 20;
static __device__ __align__(256) float g_attn_bwd_scratch[kScratchFloats];

namespace {

// In host code the array's name is only a host-side stand-in, not a device
// address.  The device address belongs to the module as loaded into the
// current context, so it is looked up again (cudaGetSymbolAddress, which
// allocates nothing) on every call made outside stream capture: after a
// cudaDeviceReset, or with another context current, the fresh value is used.
// Inside a stream capture the value recorded by the last uncaptured call on
// that device is used; a capture with no earlier call on the device fails.
constexpr int kMaxDevices = 64;
std::atomic<float*> g_scratch_dev[kMaxDevices];

}  // namespace

extern "C" int gpt2_op_attention_bwd_bf16_noalloc(const uint16_t* qkv, const uint16_t* o, const float* lse,
                                                  const uint16_t* dout, uint16_t* dqkv, int B, int T, int H,
                                                  int hd, void* stream) {
  if (!qkv || !o || !lse || !dout || !dqkv || B < 0 || T < 0 || H < 1 || hd < 1) return GPT2_ERR_INVALID_ARG;
  // the same shape rule as the entry point that takes caller scratch, checked
  // before the scratch size so the two report the same error for a bad head size
  if (hd != 16 && hd != 64) return GPT2_ERR_UNSUPPORTED_SHAPE;
  const size_t need = (size_t)B * T * H * hd + (size_t)B * H * T;
  if (need > kScratchFloats) return GPT2_ERR_TOO_LARGE;
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int dev = 0;
  CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices) return GPT2_ERR_INVALID_ARG;
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  CUDA_TRY(cudaStreamIsCapturing(st, &cap));
  float* base = nullptr;
  if (cap == cudaStreamCaptureStatusNone) {
    void* p = nullptr;
    CUDA_TRY(cudaGetSymbolAddress(&p, g_attn_bwd_scratch));
    base = static_cast<float*>(p);
    g_scratch_dev[dev].store(base, std::memory_order_relaxed);
  } else {
    base = g_scratch_dev[dev].load(std::memory_order_relaxed);
    if (!base) return GPT2_ERR_BAD_STATE;
  }
  // The backward's first kernel zeroes the dQ accumulator rows it uses and
  // overwrites D, so whatever an earlier call left in the array is harmless.
  float* dq_acc = base;
  float* dvec = dq_acc + (size_t)B * T * H * hd;
  return attn_bwd_bf16(qkv, o, lse, dout, dqkv, dq_acc, dvec, B, T, H, hd, st);
}
