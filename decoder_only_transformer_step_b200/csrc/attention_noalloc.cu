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
#include "common.cuh"
#include "internal.h"

// dQ accumulator (B*T*H*hd floats) followed by D (B*H*T floats).
static constexpr size_t kScratchFloats = size_t(4) << 20;
static __device__ __align__(256) float g_attn_bwd_scratch[kScratchFloats];

namespace {

// In host code the array's name is only a host-side stand-in, not a device
// address: the device address is looked up once per device, with that device
// current, and cached here.
constexpr int kMaxDevices = 64;
float* g_scratch_dev[kMaxDevices] = {};

}  // namespace

extern "C" int gpt2_op_attention_bwd_bf16_noalloc(const uint16_t* qkv, const uint16_t* o, const float* lse,
                                                  const uint16_t* dout, uint16_t* dqkv, int B, int T, int H,
                                                  int hd, void* stream) {
  if (!qkv || !o || !lse || !dout || !dqkv || B < 0 || T < 0 || H < 1) return GPT2_ERR_INVALID_ARG;
  const size_t need = (size_t)B * T * H * hd + (size_t)B * H * T;
  if (need > kScratchFloats) return GPT2_ERR_TOO_LARGE;
  int dev = 0;
  CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices) return GPT2_ERR_INVALID_ARG;
  if (!g_scratch_dev[dev]) {
    void* p = nullptr;
    CUDA_TRY(cudaGetSymbolAddress(&p, g_attn_bwd_scratch));
    g_scratch_dev[dev] = static_cast<float*>(p);
  }
  // The backward's first kernel zeroes the dQ accumulator rows it uses and
  // overwrites D, so whatever an earlier call left in the array is harmless.
  float* dq_acc = g_scratch_dev[dev];
  float* dvec = dq_acc + (size_t)B * T * H * hd;
  return attn_bwd_bf16(qkv, o, lse, dout, dqkv, dq_acc, dvec, B, T, H, hd,
                       reinterpret_cast<cudaStream_t>(stream));
}
