// moe_router_topk_noalloc: the router (fp32 logits, sigmoid, noaux_tc biased
// top-k, normalisation, routed scaling) without any device allocation.
//
// Who needs it: callers that cannot call cudaMalloc. A serving engine often
// reserves nearly all of the GPU's memory for its own pool at start-up, so a
// library allocation either fails or eats into that pool; and cudaMalloc can
// synchronise the device, which a latency-critical step cannot afford. Such a
// caller passes its own inputs and outputs, and the router's scratch (the
// split-K partial logits, the per-expert counters and token bitmaps) lives in
// the file-scope device array below, which exists once per GPU for as long as
// the library stays loaded.
//
// The array is shared by every call on a GPU and keeps the last call's
// contents. Each call clears the parts that must start at zero (counters,
// bitmaps, status word); the partial logits are fully overwritten. Two calls
// whose work overlaps on the GPU (different streams without ordering, or
// several host threads) race on the array and must not be issued.
// The top-k kernel's status word (set for NaN keys, which then get the
// smallest untaken expert ids) lives in the array too and is not read back:
// this call returns without waiting for the GPU, so it reports host-side
// argument errors only.
#include <cuda_runtime.h>

#include <mutex>

#include "internal.h"

namespace {

constexpr size_t kScratchBytes = size_t(16) << 20;  // 16 MiB
constexpr int kMaxDevices = 64;

// Scratch of the no-allocation router. Host code must not use this name as a
// device address: it takes the address from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_router_scratch[kScratchBytes];

std::mutex g_setup_mutex;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device; looked up once
// per device, on the first call that runs there.
cudaError_t scratch_address(int dev, void** out) {
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_router_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

size_t round256(size_t b) { return (b + 255) & ~size_t(255); }

}  // namespace

extern "C" moe_status_t moe_router_topk_noalloc(const void* x, int64_t T,
                                                const float* router_weight,
                                                const float* e_score_correction_bias,
                                                int32_t hidden_size, int32_t n_routed_experts,
                                                int32_t num_experts_per_tok,
                                                int32_t norm_topk_prob,
                                                float routed_scaling_factor, int32_t* topk_ids,
                                                float* topk_weights, void* stream) {
  if (x == nullptr || router_weight == nullptr || e_score_correction_bias == nullptr ||
      topk_ids == nullptr || topk_weights == nullptr)
    return MOE_ERR_INVALID_ARG;
  if (T < 0 || hidden_size <= 0 || n_routed_experts <= 0 || num_experts_per_tok <= 0 ||
      num_experts_per_tok > n_routed_experts || (norm_topk_prob != 0 && norm_topk_prob != 1) ||
      !(routed_scaling_factor > 0.f))
    return MOE_ERR_INVALID_ARG;
  if (hidden_size % smoe::kRouterKTile != 0 || n_routed_experts > smoe::kMaxExperts ||
      num_experts_per_tok > smoe::kMaxTopK)
    return MOE_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(router_weight)) & 15)
    return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  // the partial logits alone take 4 * T * E bytes: larger T cannot fit, and
  // rejecting it here keeps the size arithmetic below far from overflow
  if (T > static_cast<int64_t>(kScratchBytes / (4 * static_cast<size_t>(n_routed_experts))))
    return MOE_ERR_INVALID_ARG;

  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_ERR_CUDA;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return MOE_ERR_CUDA;

  // layout: [status | counts[E] | bitmaps[E][W] | partial logits[splits][T][E]]
  const size_t E = static_cast<size_t>(n_routed_experts);
  const size_t W = (static_cast<size_t>(T) + 31) / 32;
  const size_t zero_bytes = round256(256 + E * 4 + E * W * 4);
  smoe::Dims dm{};
  dm.d = hidden_size;
  dm.E = n_routed_experts;
  int splits = smoe::router_splits(dm, T, sms);
  auto need = [&](int sp) { return zero_bytes + static_cast<size_t>(sp) * T * E * 4; };
  while (splits > 1 && need(splits) > kScratchBytes) --splits;
  if (need(splits) > kScratchBytes) return MOE_ERR_INVALID_ARG;  // T * E too large for 16 MiB
  {  // a reduced count: slices of a multiple of 32 columns, none of them empty
    const int kps = ((hidden_size + splits - 1) / splits + 31) / 32 * 32;
    splits = (hidden_size + kps - 1) / kps;
  }

  void* base = nullptr;
  if (scratch_address(dev, &base) != cudaSuccess) return MOE_ERR_CUDA;
  unsigned char* b = static_cast<unsigned char*>(base);
  uint32_t* status = reinterpret_cast<uint32_t*>(b);
  int32_t* counts = reinterpret_cast<int32_t*>(b + 256);
  uint32_t* bitmap = reinterpret_cast<uint32_t*>(b + 256 + E * 4);
  float* part = reinterpret_cast<float*>(b + zero_bytes);

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(b, 0, zero_bytes, s) != cudaSuccess) return MOE_ERR_CUDA;
  cudaError_t e = smoe::launch_router_raw(
      x, router_weight, e_score_correction_bias, static_cast<int>(T), hidden_size,
      n_routed_experts, num_experts_per_tok, routed_scaling_factor, norm_topk_prob, splits, part,
      counts, bitmap, static_cast<int>(W), status, topk_ids, topk_weights, s);
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
