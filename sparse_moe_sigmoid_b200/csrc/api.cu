// C ABI of the K2 MoE layer (declared in include/moe.h): configuration
// checks, device buffers, TMA descriptors, weight loading and the forward
// sequence
//   router logits -> top-k -> route scan -> dispatch -> gate/up GEMM
//   -> down GEMM -> combine
// on one stream with no host synchronisation.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdio.h>
#include <string.h>

#include <new>
#include <string>

#include "internal.h"

using smoe::Dims;
using smoe::GemmPlan;

namespace smoe {

int bn_index(int bn) { return (bn >= 16 && bn <= 256 && bn % 16 == 0) ? bn / 16 - 1 : -1; }

using EncodeTiledFn = decltype(&cuTensorMapEncodeTiled);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

bool make_tmap(CUtensorMap* m, CUtensorMapDataType dt, int rank, void* base,
               const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box,
               std::string* err) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) {
    *err = "cuTensorMapEncodeTiled not available from the driver";
    return false;
  }
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(m, dt, static_cast<cuuint32_t>(rank), base,
                  reinterpret_cast<const cuuint64_t*>(dims),
                  reinterpret_cast<const cuuint64_t*>(strides_bytes),
                  reinterpret_cast<const cuuint32_t*>(box), estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    char buf[96];
    snprintf(buf, sizeof buf, "cuTensorMapEncodeTiled failed (CUresult %d)", static_cast<int>(r));
    *err = buf;
    return false;
  }
  return true;
}

}  // namespace smoe

namespace {

struct DeviceGuard {
  int prev = -1;
  bool ok = true;
  explicit DeviceGuard(int dev) {
    if (cudaGetDevice(&prev) != cudaSuccess) prev = -1;
    if (prev != dev) ok = cudaSetDevice(dev) == cudaSuccess;
  }
  ~DeviceGuard() {
    int cur = -1;
    if (prev >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev) cudaSetDevice(prev);
  }
};

moe_status_t fail(moe_handle* h, moe_status_t st, const std::string& msg) {
  if (h) h->last_error = msg;
  return st;
}

moe_status_t cuda_fail(moe_handle* h, cudaError_t e, const char* what) {
  std::string m = std::string(what) + ": " + cudaGetErrorString(e);
  if (h && !h->last_error.empty() && e == cudaErrorLaunchOutOfResources)
    m += " (" + h->last_error + ")";  // the launcher's resource details
  if (h) h->last_error = m;
  return e == cudaErrorMemoryAllocation ? MOE_ERR_OOM : MOE_ERR_CUDA;
}

#define CUDA_TRY(h, expr, what)                         \
  do {                                                  \
    cudaError_t e_ = (expr);                            \
    if (e_ != cudaSuccess) return cuda_fail(h, e_, what); \
  } while (0)

template <typename T>
cudaError_t alloc(T** p, size_t bytes) {
  *p = nullptr;
  if (bytes == 0) return cudaSuccess;
  return cudaMalloc(reinterpret_cast<void**>(p), bytes);
}

moe_status_t validate(const moe_config_t* c, std::string* why) {
  auto bad = [&](const char* m) {
    *why = m;
    return MOE_ERR_INVALID_ARG;
  };
  auto unsup = [&](const char* m) {
    *why = m;
    return MOE_ERR_UNSUPPORTED;
  };
  if (c->hidden_size <= 0 || c->moe_intermediate_size <= 0 || c->n_routed_experts < 0 ||
      c->num_experts_per_tok < 0 || c->n_shared_experts < 0 || c->max_tokens <= 0)
    return bad("sizes must be positive (n_shared_experts >= 0)");
  if (c->n_routed_experts == 0) {
    // no routed experts: the layer is its shared MLP alone (a dense FFN)
    if (c->num_experts_per_tok != 0 || c->n_shared_experts < 1)
      return bad("without routed experts: num_experts_per_tok 0 and n_shared_experts >= 1");
  } else if (c->num_experts_per_tok <= 0) {
    return bad("num_experts_per_tok must be positive");
  }
  if (c->num_experts_per_tok > c->n_routed_experts)
    return bad("num_experts_per_tok > n_routed_experts");
  if (c->hidden_size % 128 || c->moe_intermediate_size % 128)
    return unsup("hidden_size and moe_intermediate_size must be multiples of 128");
  if (c->hidden_size > 16384 || c->moe_intermediate_size > 8192)
    return unsup("hidden_size <= 16384 and moe_intermediate_size <= 8192");
  if (c->n_routed_experts > smoe::kMaxExperts) return unsup("n_routed_experts > 512");
  if (c->num_experts_per_tok > smoe::kMaxTopK) return unsup("num_experts_per_tok > 32");
  if (c->n_shared_experts > 16) return unsup("n_shared_experts > 16");
  if (c->n_group < 1 || c->topk_group < 1 || c->topk_group > c->n_group)
    return bad("need 1 <= topk_group <= n_group");
  if (c->n_routed_experts == 0 && (c->n_group != 1 || c->topk_group != 1))
    return bad("without routed experts: n_group = topk_group = 1");
  if (c->n_group > 32) return unsup("n_group > 32");
  if (c->n_routed_experts > 0 && c->n_routed_experts % c->n_group)
    return bad("n_group must divide n_routed_experts");
  if (c->n_routed_experts > 0 &&
      c->num_experts_per_tok > c->topk_group * (c->n_routed_experts / c->n_group))
    return bad("num_experts_per_tok exceeds the experts of topk_group groups");
  if (c->scoring_func != MOE_SCORING_SIGMOID) return unsup("scoring_func must be sigmoid");
  if (c->topk_method != MOE_TOPK_NOAUX_TC) return unsup("topk_method must be noaux_tc");
  if (c->norm_topk_prob != 0 && c->norm_topk_prob != 1) return bad("norm_topk_prob is 0 or 1");
  if (!(c->routed_scaling_factor > 0.f)) return bad("routed_scaling_factor must be > 0");
  if (c->weight_format != MOE_WEIGHT_BF16 && c->weight_format != MOE_WEIGHT_FP8_E4M3_BLOCK)
    return unsup("unknown weight_format");
  if (c->weight_format == MOE_WEIGHT_FP8_E4M3_BLOCK &&
      (c->weight_block_size[0] != 128 || c->weight_block_size[1] != 128))
    return unsup("FP8 weights need weight_block_size {128, 128}");
  if (c->weight_format == MOE_WEIGHT_FP8_E4M3_BLOCK &&
      c->activation_scheme != MOE_ACTIVATION_DYNAMIC)
    return unsup("FP8 needs activation_scheme dynamic");
  if (c->weight_format == MOE_WEIGHT_FP8_E4M3_BLOCK &&
      (c->hidden_size > 8192 || c->moe_intermediate_size > 8192))
    return unsup("FP8: hidden_size and moe_intermediate_size <= 8192");
  const int64_t rows = c->max_tokens * (c->num_experts_per_tok + c->n_shared_experts);
  if (c->max_tokens > (1 << 20) || rows > (int64_t(1) << 30))
    return unsup("max_tokens too large (at most 2^20 tokens)");
  if (c->single_launch_max_tokens < 0) return bad("single_launch_max_tokens must be >= 0");
  return MOE_OK;
}

void free_all(moe_handle* h) {
  auto f = [](void* p) {
    if (p) cudaFree(p);
  };
  f(h->w.router); f(h->w.router_cat); f(h->w.bias); f(h->w.gate); f(h->w.up); f(h->w.down);
  f(h->w.gate_s); f(h->w.up_s); f(h->w.down_s);
  f(h->ws.logits_part); f(h->ws.ids); f(h->ws.wts); f(h->ws.sched); f(h->ws.word_prefix);
  f(h->ws.offsets); f(h->ws.unit_base); f(h->ws.pair_row); f(h->ws.row_token); f(h->ws.xp);
  f(h->ws.xs); f(h->ws.hbuf); f(h->ws.hs); f(h->ws.out); f(h->ws.status);
  for (int b = 0; b < 2; ++b) {
    f(h->ws.x_stage[b]);
    f(h->ws.y_stage[b]);
    if (h->ev_x[b]) cudaEventDestroy(h->ev_x[b]);
    if (h->ev_fwd[b]) cudaEventDestroy(h->ev_fwd[b]);
    if (h->ev_y[b]) cudaEventDestroy(h->ev_y[b]);
    h->ev_x[b] = h->ev_fwd[b] = h->ev_y[b] = nullptr;
  }
  if (h->up) cudaStreamDestroy(h->up);
  if (h->down) cudaStreamDestroy(h->down);
  h->up = h->down = nullptr;
  for (auto& g : h->graphs) {
    if (g.exec) cudaGraphExecDestroy(g.exec);
    g = moe_handle::Graph{};
  }
  if (h->cap) cudaStreamDestroy(h->cap);
  if (h->ev_in) cudaEventDestroy(h->ev_in);
  if (h->ev_out) cudaEventDestroy(h->ev_out);
  h->cap = nullptr;
  h->ev_in = h->ev_out = nullptr;
  for (cudaEvent_t e : h->prof_events) cudaEventDestroy(e);
  h->prof_events.clear();
  if (h->prof_stamps) cudaFree(h->prof_stamps);
  h->prof_stamps = nullptr;
}

}  // namespace

extern "C" {

moe_status_t moe_config_init_k2(moe_config_t* c) {
  if (c == nullptr) return MOE_ERR_INVALID_ARG;
  memset(c, 0, sizeof *c);
  c->hidden_size = 7168;
  c->moe_intermediate_size = 2048;
  c->n_routed_experts = 384;
  c->num_experts_per_tok = 8;
  c->n_shared_experts = 1;
  c->n_group = 1;
  c->topk_group = 1;
  c->norm_topk_prob = 1;
  c->routed_scaling_factor = 2.827f;
  c->scoring_func = MOE_SCORING_SIGMOID;
  c->topk_method = MOE_TOPK_NOAUX_TC;
  c->weight_format = MOE_WEIGHT_BF16;
  c->weight_block_size[0] = 128;
  c->weight_block_size[1] = 128;
  c->activation_scheme = MOE_ACTIVATION_DYNAMIC;
  c->max_tokens = 8192;
  c->single_launch_max_tokens = 0;
  return MOE_OK;
}

moe_status_t moe_create(const moe_config_t* cfg, int device, moe_handle_t** out) {
  if (cfg == nullptr || out == nullptr) return MOE_ERR_INVALID_ARG;
  *out = nullptr;
  std::string why;
  moe_status_t st = validate(cfg, &why);
  if (st != MOE_OK) return st;
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess || device < 0 || device >= ndev)
    return MOE_ERR_INVALID_ARG;
  DeviceGuard guard(device);
  if (!guard.ok) return MOE_ERR_CUDA;
  cudaDeviceProp prop;
  if (cudaGetDeviceProperties(&prop, device) != cudaSuccess) return MOE_ERR_CUDA;
  if (prop.major != 10) return MOE_ERR_UNSUPPORTED;  // sm_100a kernels only

  moe_handle* h = new (std::nothrow) moe_handle();
  if (h == nullptr) return MOE_ERR_OOM;
  h->cfg = *cfg;
  h->device = device;
  h->num_sms = prop.multiProcessorCount;
  Dims& dm = h->dims;
  dm.d = cfg->hidden_size;
  dm.f = cfg->moe_intermediate_size;
  dm.E = cfg->n_routed_experts;
  dm.k = cfg->num_experts_per_tok;
  dm.ns = cfg->n_shared_experts;
  dm.G = dm.E + dm.ns;
  dm.fp8 = cfg->weight_format == MOE_WEIGHT_FP8_E4M3_BLOCK;
  dm.Tmax = cfg->max_tokens;
  dm.Rmax = dm.Tmax * (dm.k + dm.ns);
  const size_t wb = dm.fp8 ? 1 : 2;  // bytes per weight / activation operand value
  const size_t d = dm.d, f = dm.f, E = dm.E, G = dm.G;
  const size_t Tm = dm.Tmax, Rm = dm.Rmax;
  const size_t W = (Tm + 31) / 32;

  // the router's split-K partial buffer: largest splits(T) * T over T <= Tmax
  size_t part_rows = 0;
  for (int64_t T = 64; dm.E > 0; T += 64) {
    const int64_t Tc = T < dm.Tmax ? T : dm.Tmax;
    const int sp = Tc >= smoe::kTensorRouterMinT ? smoe::kTensorRouterSplits
                                                 : smoe::router_splits(dm, Tc, h->num_sms);
    const size_t rows = static_cast<size_t>(sp) * Tc;
    if (rows > part_rows) part_rows = rows;
    if (Tc == dm.Tmax) break;
  }

  moe_status_t rc = MOE_OK;
  auto A = [&](auto** p, size_t bytes, const char* what) {
    if (rc != MOE_OK) return;
    cudaError_t e = alloc(p, bytes);
    if (e != cudaSuccess) rc = cuda_fail(h, e, what);
  };
  A(&h->w.router, E * d * 4, "router weight");
  A(&h->w.router_cat, E * 3 * d * 2, "router weight split");
  A(&h->w.bias, E * 4, "bias");
  A(&h->w.gate, G * f * d * wb, "gate_proj");
  A(&h->w.up, G * f * d * wb, "up_proj");
  A(&h->w.down, G * d * f * wb, "down_proj");
  if (dm.fp8) {
    A(&h->w.gate_s, G * (f / 128) * (d / 128) * 4, "gate scales");
    A(&h->w.up_s, G * (f / 128) * (d / 128) * 4, "up scales");
    A(&h->w.down_s, G * (d / 128) * (f / 128) * 4, "down scales");
  }
  A(&h->ws.logits_part, part_rows * E * 4, "router partials");
  A(&h->ws.ids, Tm * dm.k * 4, "ids");
  A(&h->ws.wts, Tm * dm.k * 4, "weights");
  // zeroed at the start of every forward: [unit counters | counts | bitmaps |
  // single-launch sync words]
  h->ws.zero_bytes = 256 + E * 4 + E * W * 4 + (2 + G) * 4;
  {
    void* z = nullptr;
    A(&z, h->ws.zero_bytes, "counts/bitmap");
    char* zc = static_cast<char*>(z);
    h->ws.sched = static_cast<int32_t*>(z);
    h->ws.counts = z ? reinterpret_cast<int32_t*>(zc + 256) : nullptr;
    h->ws.bitmap = z ? reinterpret_cast<uint32_t*>(zc + 256 + E * 4) : nullptr;
    h->ws.sync = z ? reinterpret_cast<uint32_t*>(zc + 256 + E * 4 + E * W * 4) : nullptr;
  }
  A(&h->ws.word_prefix, E * W * 4, "word prefix");
  A(&h->ws.offsets, (G + 1) * 4, "offsets");
  A(&h->ws.unit_base, 2 * (G + 1) * 4, "unit prefix");
  A(&h->ws.pair_row, Tm * dm.k * 4, "pair rows");
  A(&h->ws.row_token, Rm * 4, "row tokens");
  A(&h->ws.xp, Rm * d * wb, "gathered x");
  A(&h->ws.hbuf, Rm * f * wb, "h");
  if (dm.fp8) {
    A(&h->ws.xs, Rm * (d / 128) * 4, "x scales");
    A(&h->ws.hs, Rm * (f / 128) * 4, "h scales");
  }
  A(&h->ws.out, Rm * d * 2, "expert outputs");
  A(&h->ws.status, 4, "status");
  for (int b = 0; b < 2; ++b) {
    A(&h->ws.x_stage[b], Tm * d * 2, "x staging");
    A(&h->ws.y_stage[b], Tm * d * 2, "y staging");
  }
  if (rc == MOE_OK) {
    bool ok = cudaStreamCreateWithFlags(&h->up, cudaStreamNonBlocking) == cudaSuccess &&
              cudaStreamCreateWithFlags(&h->down, cudaStreamNonBlocking) == cudaSuccess &&
              cudaStreamCreateWithFlags(&h->cap, cudaStreamNonBlocking) == cudaSuccess &&
              cudaEventCreateWithFlags(&h->ev_in, cudaEventDisableTiming) == cudaSuccess &&
              cudaEventCreateWithFlags(&h->ev_out, cudaEventDisableTiming) == cudaSuccess;
    for (int b = 0; b < 2 && ok; ++b)
      ok = cudaEventCreateWithFlags(&h->ev_x[b], cudaEventDisableTiming) == cudaSuccess &&
           cudaEventCreateWithFlags(&h->ev_fwd[b], cudaEventDisableTiming) == cudaSuccess &&
           cudaEventCreateWithFlags(&h->ev_y[b], cudaEventDisableTiming) == cudaSuccess;
    if (!ok) rc = MOE_ERR_CUDA;
  }
  if (rc != MOE_OK) {
    free_all(h);
    delete h;
    return rc;
  }
  if (cudaMemset(h->ws.status, 0, 4) != cudaSuccess) {
    free_all(h);
    delete h;
    return MOE_ERR_CUDA;
  }

  // TMA descriptors (128-byte swizzle, K innermost)
  const CUtensorMapDataType dt = dm.fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                        : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const uint32_t kbox = dm.fp8 ? 128 : 64;  // 128 bytes of K per row
  bool ok = true;
  {
    uint64_t dims[3] = {d, f, G};
    uint64_t str[2] = {d * wb, f * d * wb};
    uint32_t box[3] = {kbox, 128, 1};
    ok = ok && smoe::make_tmap(&h->tm_gate, dt, 3, h->w.gate, dims, str, box, &why);
    ok = ok && smoe::make_tmap(&h->tm_up, dt, 3, h->w.up, dims, str, box, &why);
  }
  {
    uint64_t dims[3] = {f, d, G};
    uint64_t str[2] = {f * wb, d * f * wb};
    uint32_t box[3] = {kbox, 128, 1};
    ok = ok && smoe::make_tmap(&h->tm_down, dt, 3, h->w.down, dims, str, box, &why);
  }
  {
    uint64_t dims[3] = {3 * d, E, 1};
    uint64_t str[2] = {3 * d * 2, E * 3 * d * 2};
    uint32_t box[3] = {64, 128, 1};
    ok = ok && (E == 0 || smoe::make_tmap(&h->tm_router, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                                          h->w.router_cat, dims, str, box, &why));
  }
  for (int i = 0; i < 16 && ok; ++i) {
    const uint32_t bn = 16u * (i + 1);
    uint32_t box[2] = {kbox, bn};
    uint64_t dx[2] = {d, Rm};
    uint64_t sx[1] = {d * wb};
    ok = ok && smoe::make_tmap(&h->tm_xp[i], dt, 2, h->ws.xp, dx, sx, box, &why);
    uint64_t dh[2] = {f, Rm};
    uint64_t sh[1] = {f * wb};
    ok = ok && smoe::make_tmap(&h->tm_h[i], dt, 2, h->ws.hbuf, dh, sh, box, &why);
  }
  if (dm.fp8 && ok) {  // gathers of quantised token rows, rows [0, T) of xp (one-row box)
    uint64_t dx[2] = {d, Rm};
    uint64_t sx[1] = {d};
    uint32_t box[2] = {kbox, 1};
    ok = smoe::make_tmap(&h->tm_xg, dt, 2, h->ws.xp, dx, sx, box, &why);
  }
  if (!ok) {
    free_all(h);
    delete h;
    return MOE_ERR_CUDA;
  }
  *out = h;
  return MOE_OK;
}

moe_status_t moe_load_weights(moe_handle_t* h, const moe_weights_t* w, void* stream) {
  if (h == nullptr || w == nullptr) return MOE_ERR_INVALID_ARG;
  const Dims& dm = h->dims;
  if (dm.E > 0 && (!w->router_weight || !w->e_score_correction_bias || !w->gate_proj ||
                   !w->up_proj || !w->down_proj))
    return fail(h, MOE_ERR_INVALID_ARG, "router, bias and routed expert weights are required");
  if (dm.ns > 0 && (!w->shared_gate_proj || !w->shared_up_proj || !w->shared_down_proj))
    return fail(h, MOE_ERR_INVALID_ARG, "shared expert weights are required");
  if (dm.fp8 && ((dm.E > 0 && (!w->gate_scale || !w->up_scale || !w->down_scale)) ||
                 (dm.ns > 0 && (!w->shared_gate_scale || !w->shared_up_scale ||
                                !w->shared_down_scale))))
    return fail(h, MOE_ERR_INVALID_ARG, "FP8 weights need every block-scale tensor");
  DeviceGuard guard(h->device);
  if (!guard.ok) return fail(h, MOE_ERR_CUDA, "cudaSetDevice failed");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t wb = dm.fp8 ? 1 : 2;
  const size_t d = dm.d, f = dm.f, E = dm.E, fs = f * dm.ns;
  const cudaMemcpyKind K = cudaMemcpyDefault;
  auto bytes_at = [](const void* p, size_t off) {
    return static_cast<const char*>(p) + off;
  };
  auto bytes_to = [](void* p, size_t off) { return static_cast<char*>(p) + off; };

  const size_t nb_f = f / 128, nb_d = d / 128, nb_fs = fs / 128;
  if (E > 0) {  // router and routed experts (none in a dense FFN layer)
    CUDA_TRY(h, cudaMemcpyAsync(h->w.router, w->router_weight, E * d * 4, K, s), "router copy");
    CUDA_TRY(h, cudaMemcpyAsync(h->w.bias, w->e_score_correction_bias, E * 4, K, s), "bias copy");
    CUDA_TRY(h, smoe::launch_router_split(h, s), "router split launch");
    CUDA_TRY(h, cudaMemcpyAsync(h->w.gate, w->gate_proj, E * f * d * wb, K, s), "gate copy");
    CUDA_TRY(h, cudaMemcpyAsync(h->w.up, w->up_proj, E * f * d * wb, K, s), "up copy");
    CUDA_TRY(h, cudaMemcpyAsync(h->w.down, w->down_proj, E * d * f * wb, K, s), "down copy");
    if (dm.fp8) {
      CUDA_TRY(h, cudaMemcpyAsync(h->w.gate_s, w->gate_scale, E * nb_f * nb_d * 4, K, s), "scales");
      CUDA_TRY(h, cudaMemcpyAsync(h->w.up_s, w->up_scale, E * nb_f * nb_d * 4, K, s), "scales");
      CUDA_TRY(h, cudaMemcpyAsync(h->w.down_s, w->down_scale, E * nb_d * nb_f * 4, K, s),
               "scales");
    }
  }
  // shared expert of intermediate fs = ns * f -> ns groups of f: gate/up take
  // row slices, down takes column slices (a pitched copy)
  for (int sgi = 0; sgi < dm.ns; ++sgi) {
    const size_t g = E + sgi;
    CUDA_TRY(h, cudaMemcpyAsync(bytes_to(h->w.gate, g * f * d * wb),
                                bytes_at(w->shared_gate_proj, sgi * f * d * wb), f * d * wb, K, s),
             "shared gate copy");
    CUDA_TRY(h, cudaMemcpyAsync(bytes_to(h->w.up, g * f * d * wb),
                                bytes_at(w->shared_up_proj, sgi * f * d * wb), f * d * wb, K, s),
             "shared up copy");
    CUDA_TRY(h, cudaMemcpy2DAsync(bytes_to(h->w.down, g * d * f * wb), f * wb,
                                  bytes_at(w->shared_down_proj, sgi * f * wb), fs * wb, f * wb, d,
                                  K, s),
             "shared down copy");
    if (dm.fp8) {
      CUDA_TRY(h, cudaMemcpyAsync(h->w.gate_s + g * nb_f * nb_d,
                                  w->shared_gate_scale + sgi * nb_f * nb_d, nb_f * nb_d * 4, K, s),
               "shared scales");
      CUDA_TRY(h, cudaMemcpyAsync(h->w.up_s + g * nb_f * nb_d,
                                  w->shared_up_scale + sgi * nb_f * nb_d, nb_f * nb_d * 4, K, s),
               "shared scales");
      CUDA_TRY(h, cudaMemcpy2DAsync(h->w.down_s + g * nb_d * nb_f, nb_f * 4,
                                    w->shared_down_scale + sgi * nb_f, nb_fs * 4, nb_f * 4, nb_d,
                                    K, s),
               "shared down scales");
    }
  }
  h->w.loaded = true;
  return MOE_OK;
}

static moe_status_t read_status(moe_handle* h, cudaStream_t s, uint32_t* flags) {
  uint32_t v = 0;
  CUDA_TRY(h, cudaMemcpyAsync(&v, h->ws.status, 4, cudaMemcpyDeviceToHost, s), "status read");
  CUDA_TRY(h, cudaStreamSynchronize(s), "stream sync");
  if (v != 0) CUDA_TRY(h, cudaMemsetAsync(h->ws.status, 0, 4, s), "status clear");
  CUDA_TRY(h, cudaStreamSynchronize(s), "stream sync");
  *flags = v;
  return MOE_OK;
}

namespace {
moe_status_t launch_forward(moe_handle* h, const void* x, int64_t T, void* y,
                            const moe_forward_opts_t* opts, cudaStream_t s, cudaEvent_t* ev);
moe_status_t forward_graphed(moe_handle* h, const void* x, int64_t T, void* y, cudaStream_t s);
}  // namespace

moe_status_t moe_forward(moe_handle_t* h, const void* x, int64_t T, void* y,
                         const moe_forward_opts_t* opts, void* stream) {
  if (h == nullptr) return MOE_ERR_INVALID_ARG;
  if (!h->w.loaded) return fail(h, MOE_ERR_STATE, "moe_load_weights has not been called");
  if (T < 0 || T > h->dims.Tmax) return fail(h, MOE_ERR_INVALID_ARG, "T outside [0, max_tokens]");
  if (T == 0) return MOE_OK;
  if (x == nullptr || y == nullptr) return fail(h, MOE_ERR_INVALID_ARG, "x and y are required");
  const Dims& dm = h->dims;
  const size_t nbytes = static_cast<size_t>(T) * dm.d * 2;
  const char* xb = static_cast<const char*>(x);
  const char* yb = static_cast<const char*>(y);
  if (xb < yb + nbytes && yb < xb + nbytes)
    return fail(h, MOE_ERR_INVALID_ARG, "x and y overlap");
  if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(y)) & 15)
    return fail(h, MOE_ERR_INVALID_ARG, "x and y must be 16-byte aligned");
  if (opts && (opts->reserved != 0 ||
               (opts->flags & ~(MOE_FLAG_SYNC_CHECK | MOE_FLAG_TEST_STALL | MOE_FLAG_PHASE_KERNELS))))
    return fail(h, MOE_ERR_INVALID_ARG, "unknown option flags, or reserved != 0");
  DeviceGuard guard(h->device);
  if (!guard.ok) return fail(h, MOE_ERR_CUDA, "cudaSetDevice failed");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaEvent_t* ev = nullptr;
  if (h->prof_next < h->prof_cap)
    ev = h->prof_events.data() + static_cast<size_t>(h->prof_next) * (MOE_NUM_PHASES + 1);
  if (opts == nullptr && ev == nullptr) return forward_graphed(h, x, T, y, s);
  return launch_forward(h, x, T, y, opts, s, ev);
}

namespace {

// The launch sequence of one forward on stream s (ev: per-phase events, or
// NULL).
moe_status_t launch_forward(moe_handle* h, const void* x, int64_t T, void* y,
                            const moe_forward_opts_t* opts, cudaStream_t s, cudaEvent_t* ev) {
  const Dims& dm = h->dims;
  const int Ti = static_cast<int>(T);
  auto mark = [&](int i) {
    if (ev) cudaEventRecord(ev[i], s);
  };

  const GemmPlan p1 = smoe::plan_gate_up(dm, T);
  const GemmPlan p2 = smoe::plan_down(dm, T);
  const int splits = dm.E == 0                       ? 0
                     : T <= smoe::kRouterGemvMaxT ? 1  // the GEMV router: one slice
                                                  : smoe::router_splits(dm, T, h->num_sms);
  const int32_t* forced = opts ? opts->forced_topk_ids : nullptr;
  h->fwd_wait_ns = opts ? opts->wait_limit_ns : 0;
  h->fwd_stall = opts && (opts->flags & MOE_FLAG_TEST_STALL);
  struct Reset {  // the next forward starts from the defaults again
    moe_handle* h;
    ~Reset() {
      h->fwd_wait_ns = 0;
      h->fwd_stall = false;
    }
  } reset{h};

  if (!dm.fp8 && p1.gather) {  // the gate/up GEMM gathers token rows straight from x
    uint64_t dx[2] = {static_cast<uint64_t>(dm.d), static_cast<uint64_t>(T)};
    uint64_t sx[1] = {static_cast<uint64_t>(dm.d) * 2};
    uint32_t box[2] = {64, 1};
    std::string why;
    if (!smoe::make_tmap(&h->tm_xg, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(x), dx,
                         sx, box, &why))
      return fail(h, MOE_ERR_CUDA, why);
  }

  const bool small = smoe::small_layer_supported(dm, T, h->cfg.single_launch_max_tokens) &&
                     !(opts && (opts->flags & MOE_FLAG_PHASE_KERNELS));
  if (small) {
    // the whole layer in one cooperative launch; with profiling, its phase
    // boundaries come from device timestamps
    uint64_t* stamps = nullptr;
    if (ev) {
      stamps = h->prof_stamps + static_cast<size_t>(h->prof_next) * (MOE_NUM_PHASES + 1);
      h->prof_small[h->prof_next] = 1;
    }
    mark(0);
    CUDA_TRY(h, cudaMemsetAsync(h->ws.sched, 0, h->ws.zero_bytes, s), "clear counts");
    CUDA_TRY(h,
             smoe::launch_small_layer(h, x, Ti, y, forced, opts ? opts->topk_ids_out : nullptr,
                                      opts ? opts->topk_weights_out : nullptr,
                                      opts ? opts->router_logits_out : nullptr, stamps, s),
             "single-launch layer");
    for (int i = 1; i <= MOE_NUM_PHASES; ++i) mark(i);
    if (ev) h->prof_next++;
  } else {
    if (ev) h->prof_small[h->prof_next] = 0;
    mark(0);
    CUDA_TRY(h, cudaMemsetAsync(h->ws.sched, 0, h->ws.zero_bytes, s), "clear counts");
    // without routed experts (a dense FFN layer) there is nothing to route: the
    // router phases are empty and the shared groups take every token
    const bool tensor_router = T >= smoe::kTensorRouterMinT;
    if (dm.E > 0) {
      if (tensor_router) {
        CUDA_TRY(h, smoe::launch_router_gemm(h, x, Ti, s), "router GEMM launch");
      } else {
        CUDA_TRY(h, smoe::launch_router_logits(h, x, Ti, splits, s), "router logits launch");
      }
    }
    mark(1);
    if (dm.E > 0) {
      CUDA_TRY(h,
               smoe::launch_router_topk(h, Ti, tensor_router ? smoe::kTensorRouterSplits : splits,
                                        forced, s, opts ? opts->topk_ids_out : nullptr,
                                        opts ? opts->topk_weights_out : nullptr,
                                        opts ? opts->router_logits_out : nullptr),
               "router top-k launch");
    }
    mark(2);
    CUDA_TRY(h, smoe::launch_route_scan(h, Ti, p1, p2, s), "route scan launch");
    mark(3);
    CUDA_TRY(h, smoe::launch_dispatch(h, x, Ti, p1.gather, s), "dispatch launch");
    mark(4);
    if (dm.fp8) {
      CUDA_TRY(h, smoe::launch_gemm_fp8(h, true, p1, s), "gate/up GEMM launch");
    } else if (p1.pair) {
      CUDA_TRY(h, smoe::launch_gemm_bf16_pair(h, true, p1, s), "gate/up GEMM launch");
    } else {
      CUDA_TRY(h, smoe::launch_gemm_bf16(h, true, p1, s), "gate/up GEMM launch");
    }
    mark(5);
    if (dm.fp8) {
      CUDA_TRY(h, smoe::launch_gemm_fp8(h, false, p2, s), "down GEMM launch");
    } else if (p2.pair) {
      CUDA_TRY(h, smoe::launch_gemm_bf16_pair(h, false, p2, s), "down GEMM launch");
    } else {
      CUDA_TRY(h, smoe::launch_gemm_bf16(h, false, p2, s), "down GEMM launch");
    }
    mark(6);
    CUDA_TRY(h, smoe::launch_combine(h, y, Ti, s), "combine launch");
    mark(7);
    if (ev) h->prof_next++;
  }
  if (opts && opts->expert_offsets_out && dm.E > 0)
    CUDA_TRY(h, cudaMemcpyAsync(opts->expert_offsets_out, h->ws.offsets, (dm.E + 1) * 4,
                                cudaMemcpyDeviceToDevice, s),
             "offsets copy");
  if (opts && opts->pair_rows_out && dm.E > 0)
    CUDA_TRY(h, cudaMemcpyAsync(opts->pair_rows_out, h->ws.pair_row, T * dm.k * 4,
                                cudaMemcpyDeviceToDevice, s),
             "pair rows copy");

  if (opts && (opts->flags & MOE_FLAG_SYNC_CHECK)) {
    uint32_t flags = 0;
    moe_status_t st = read_status(h, s, &flags);
    if (st != MOE_OK) return st;
    if (flags & MOE_DEVICE_WAIT_TIMEOUT)
      return fail(h, MOE_ERR_TIMEOUT, "a GEMM pipeline wait ran out of time");
    if (flags) return fail(h, MOE_ERR_DEVICE, "device status word set");
  }
  return MOE_OK;
}

// A forward without options or profiling, as a CUDA graph: at small T the
// layer is a chain of short kernels and the launches themselves are a large
// part of the step. The first call with a given (T, x, y) launches directly
// (which also does each kernel's one-time attribute setup); the second
// captures the same launch sequence on the handle's capture stream, and every
// later call replays it there, ordered after the caller's stream by an event
// and with the caller's stream waiting for it.
moe_status_t forward_graphed(moe_handle* h, const void* x, int64_t T, void* y, cudaStream_t s) {
  moe_handle::Graph* g = nullptr;
  for (auto& e : h->graphs)
    if (e.T == T && e.x == x && e.y == y) g = &e;
  if (g == nullptr) {  // first sight: remember it, launch directly
    moe_handle::Graph* slot = &h->graphs[0];
    for (auto& e : h->graphs)
      if (e.last_use < slot->last_use) slot = &e;
    if (slot->exec) cudaGraphExecDestroy(slot->exec);
    *slot = moe_handle::Graph{};
    slot->T = T;
    slot->x = x;
    slot->y = y;
    slot->last_use = ++h->graph_clock;
    return launch_forward(h, x, T, y, nullptr, s, nullptr);
  }
  g->last_use = ++h->graph_clock;
  if (g->exec == nullptr && !g->failed) {  // second sight: capture
    const int64_t n0 = h->launches;
    cudaGraph_t graph = nullptr;
    bool ok = cudaStreamBeginCapture(h->cap, cudaStreamCaptureModeThreadLocal) == cudaSuccess;
    moe_status_t st = ok ? launch_forward(h, x, T, y, nullptr, h->cap, nullptr) : MOE_ERR_CUDA;
    if (ok) ok = cudaStreamEndCapture(h->cap, &graph) == cudaSuccess && st == MOE_OK;
    if (ok) ok = cudaGraphInstantiate(&g->exec, graph, 0) == cudaSuccess;
    if (graph) cudaGraphDestroy(graph);
    const int64_t captured = h->launches - n0;  // kernels in the graph
    h->launches = n0;
    if (!ok) {  // run without a graph from now on for this key
      g->failed = true;
      g->exec = nullptr;
      cudaGetLastError();
    } else {
      g->launches = captured;
    }
  }
  if (g->exec == nullptr) return launch_forward(h, x, T, y, nullptr, s, nullptr);
  CUDA_TRY(h, cudaEventRecord(h->ev_in, s), "graph order");
  CUDA_TRY(h, cudaStreamWaitEvent(h->cap, h->ev_in, 0), "graph order");
  CUDA_TRY(h, cudaGraphLaunch(g->exec, h->cap), "graph launch");
  CUDA_TRY(h, cudaEventRecord(h->ev_out, h->cap), "graph order");
  CUDA_TRY(h, cudaStreamWaitEvent(s, h->ev_out, 0), "graph order");
  h->launches += g->launches;
  return MOE_OK;
}

}  // namespace

moe_status_t moe_forward_host_async(moe_handle_t* h, const void* x_host, int64_t T, void* y_host,
                                    const moe_forward_opts_t* opts, void* stream) {
  if (h == nullptr) return MOE_ERR_INVALID_ARG;
  if (T < 0 || T > h->dims.Tmax) return fail(h, MOE_ERR_INVALID_ARG, "T outside [0, max_tokens]");
  if (T == 0) return MOE_OK;
  if (x_host == nullptr || y_host == nullptr)
    return fail(h, MOE_ERR_INVALID_ARG, "x_host and y_host are required");
  if (!h->w.loaded) return fail(h, MOE_ERR_STATE, "moe_load_weights has not been called");
  DeviceGuard guard(h->device);
  if (!guard.ok) return fail(h, MOE_ERR_CUDA, "cudaSetDevice failed");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t nbytes = static_cast<size_t>(T) * h->dims.d * 2;
  const int b = static_cast<int>(h->host_calls & 1);
  // upload into staging b once the forward that read it (two calls ago) is done
  CUDA_TRY(h, cudaStreamWaitEvent(h->up, h->ev_fwd[b], 0), "upload wait");
  CUDA_TRY(h, cudaMemcpyAsync(h->ws.x_stage[b], x_host, nbytes, cudaMemcpyHostToDevice, h->up),
           "x copy");
  CUDA_TRY(h, cudaEventRecord(h->ev_x[b], h->up), "upload event");
  // the forward on the caller's stream: after the upload, and once y staging
  // b has been downloaded (two calls ago)
  CUDA_TRY(h, cudaStreamWaitEvent(s, h->ev_x[b], 0), "forward wait");
  CUDA_TRY(h, cudaStreamWaitEvent(s, h->ev_y[b], 0), "forward wait");
  moe_status_t st = moe_forward(h, h->ws.x_stage[b], T, h->ws.y_stage[b], opts, stream);
  if (st != MOE_OK) return st;
  CUDA_TRY(h, cudaEventRecord(h->ev_fwd[b], s), "forward event");
  // download after the forward
  CUDA_TRY(h, cudaStreamWaitEvent(h->down, h->ev_fwd[b], 0), "download wait");
  CUDA_TRY(h, cudaMemcpyAsync(y_host, h->ws.y_stage[b], nbytes, cudaMemcpyDeviceToHost, h->down),
           "y copy");
  CUDA_TRY(h, cudaEventRecord(h->ev_y[b], h->down), "download event");
  ++h->host_calls;
  return MOE_OK;
}

moe_status_t moe_host_wait(moe_handle_t* h) {
  if (h == nullptr) return MOE_ERR_INVALID_ARG;
  DeviceGuard guard(h->device);
  if (!guard.ok) return fail(h, MOE_ERR_CUDA, "cudaSetDevice failed");
  CUDA_TRY(h, cudaStreamSynchronize(h->up), "upload sync");
  CUDA_TRY(h, cudaStreamSynchronize(h->down), "download sync");  // follows every forward
  return MOE_OK;
}

moe_status_t moe_forward_host(moe_handle_t* h, const void* x_host, int64_t T, void* y_host,
                              const moe_forward_opts_t* opts, void* stream) {
  moe_status_t st = moe_forward_host_async(h, x_host, T, y_host, opts, stream);
  if (st != MOE_OK || T == 0) return st;
  return moe_host_wait(h);
}

moe_status_t moe_get_device_status(moe_handle_t* h, uint32_t* flags) {
  if (h == nullptr || flags == nullptr) return MOE_ERR_INVALID_ARG;
  DeviceGuard guard(h->device);
  CUDA_TRY(h, cudaDeviceSynchronize(), "device sync");
  uint32_t v = 0;
  CUDA_TRY(h, cudaMemcpy(&v, h->ws.status, 4, cudaMemcpyDeviceToHost), "status read");
  if (v) CUDA_TRY(h, cudaMemset(h->ws.status, 0, 4), "status clear");
  *flags = v;
  return MOE_OK;
}

moe_status_t moe_profile_enable(moe_handle_t* h, int32_t max_forwards) {
  if (h == nullptr || max_forwards < 0) return MOE_ERR_INVALID_ARG;
  DeviceGuard guard(h->device);
  for (cudaEvent_t e : h->prof_events) cudaEventDestroy(e);
  h->prof_events.clear();
  h->prof_cap = 0;
  h->prof_next = 0;
  if (h->prof_stamps) cudaFree(h->prof_stamps);
  h->prof_stamps = nullptr;
  const size_t n = static_cast<size_t>(max_forwards) * (MOE_NUM_PHASES + 1);
  if (n > 0) CUDA_TRY(h, cudaMalloc(&h->prof_stamps, n * 8), "profile stamps");
  h->prof_small.assign(static_cast<size_t>(max_forwards), 0);
  h->prof_events.resize(n);
  for (size_t i = 0; i < n; ++i) {
    cudaError_t e = cudaEventCreate(&h->prof_events[i]);
    if (e != cudaSuccess) {
      h->prof_events.resize(i);
      return cuda_fail(h, e, "event create");
    }
  }
  h->prof_cap = max_forwards;
  return MOE_OK;
}

moe_status_t moe_profile_read(moe_handle_t* h, float* ms, int32_t cap, int32_t* n_forwards) {
  if (h == nullptr || n_forwards == nullptr || (ms == nullptr && cap > 0))
    return MOE_ERR_INVALID_ARG;
  DeviceGuard guard(h->device);
  const int n = h->prof_next;
  *n_forwards = n;
  for (int i = 0; i < n; ++i) {
    cudaEvent_t* ev = h->prof_events.data() + static_cast<size_t>(i) * (MOE_NUM_PHASES + 1);
    CUDA_TRY(h, cudaEventSynchronize(ev[MOE_NUM_PHASES]), "event sync");
    uint64_t st[MOE_NUM_PHASES + 1] = {};
    const bool small = h->prof_small[i] != 0;
    if (small)
      CUDA_TRY(h, cudaMemcpy(st, h->prof_stamps + static_cast<size_t>(i) * (MOE_NUM_PHASES + 1),
                             sizeof st, cudaMemcpyDeviceToHost),
               "stamps read");
    for (int p = 0; p < MOE_NUM_PHASES; ++p) {
      const int idx = i * MOE_NUM_PHASES + p;
      if (idx >= cap) return MOE_OK;
      float t = 0.f;
      if (small) t = static_cast<float>(static_cast<double>(st[p + 1] - st[p]) * 1e-6);
      else CUDA_TRY(h, cudaEventElapsedTime(&t, ev[p], ev[p + 1]), "event elapsed");
      ms[idx] = t;
    }
  }
  return MOE_OK;
}

moe_status_t moe_act_quant_e4m3(const void* x, int64_t rows, int32_t cols, void* q, float* scales,
                                void* stream) {
  if (rows < 0 || cols <= 0 || cols % 128 != 0) return MOE_ERR_INVALID_ARG;
  if (rows == 0) return MOE_OK;
  if (x == nullptr || q == nullptr || scales == nullptr) return MOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(q)) & 15)
    return MOE_ERR_INVALID_ARG;
  if (rows > (int64_t(1) << 26)) return MOE_ERR_INVALID_ARG;
  cudaError_t e = smoe::launch_act_quant(x, rows, cols, static_cast<uint8_t*>(q), scales,
                                         static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status_t moe_combine_rows(const void* pair_out, const float* weights, const void* shared_out,
                              int64_t T, int32_t hidden_size, int32_t num_experts_per_tok,
                              void* y, void* stream) {
  if (T < 0 || hidden_size <= 0 || hidden_size % 8 || num_experts_per_tok <= 0 ||
      num_experts_per_tok > smoe::kMaxTopK)
    return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (pair_out == nullptr || weights == nullptr || y == nullptr) return MOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(pair_out) | reinterpret_cast<uintptr_t>(shared_out) |
       reinterpret_cast<uintptr_t>(y)) & 15)
    return MOE_ERR_INVALID_ARG;
  if (T > (int64_t(1) << 31) - 1) return MOE_ERR_INVALID_ARG;
  cudaError_t e = smoe::launch_combine_rows(pair_out, weights, shared_out, static_cast<int>(T),
                                            hidden_size, num_experts_per_tok, y,
                                            static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

int64_t moe_launch_count(const moe_handle_t* h) { return h ? h->launches : 0; }

void moe_destroy(moe_handle_t* h) {
  if (h == nullptr) return;
  {
    DeviceGuard guard(h->device);
    cudaDeviceSynchronize();
    free_all(h);
  }
  delete h;
}

const char* moe_status_string(moe_status_t s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported configuration";
    case MOE_ERR_OOM: return "out of device memory";
    case MOE_ERR_CUDA: return "CUDA runtime error";
    case MOE_ERR_DEVICE: return "a kernel reported a problem";
    case MOE_ERR_TIMEOUT: return "a kernel wait ran out of time";
    case MOE_ERR_STATE: return "call out of order";
  }
  return "unknown status";
}

const char* moe_last_error(const moe_handle_t* h) { return h ? h->last_error.c_str() : ""; }

}  // extern "C"
