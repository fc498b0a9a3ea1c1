// Internal declarations shared by the library's .cu files (not installed).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <string>
#include <vector>

#include "../../include/moe.h"

namespace smoe {

constexpr int kBlock = 128;       // FP8 block edge and GEMM M tile
constexpr int kMaxTopK = 32;
constexpr int kMaxExperts = 512;
constexpr int kRouterTile = 64;   // router tile: 64 tokens x 64 experts
constexpr int kRouterKTile = 32;
constexpr int kRouterMaxSplits = 32;
constexpr int kRouterGemvMaxT = 8;  // up to this many tokens the logits are a GEMV (one slice)
constexpr int kSmallMaxT = 128;     // up to this many tokens the layer may run as one launch

// Sizes derived from the config, fixed per handle.
struct Dims {
  int d, f, E, k, ns, G;  // G = E + ns groups (shared expert split into ns groups)
  bool fp8;
  int64_t Tmax, Rmax;     // Rmax = Tmax * (k + ns)
};

// One grouped GEMM launch's shape choice.
struct GemmPlan {
  int bn;       // token rows per tile (MMA N upper bound)
  int na;       // weight tiles per unit (2: gate+up, or two halves of 256 features)
  bool pair;    // BF16 on CTA pairs (2-SM MMA): units of 256 output features
  int m_tiles;  // output feature tiles (128 rows each, or 256 for a plain na = 2 unit)
  int k_blocks; // reduction / kernel K step
  bool gather;  // gate/up: gather token rows from x with tile::gather4 (no row copies)
};

// Row tiles up to this height gather their B rows from x (a tile::gather4
// moves four 128-byte rows, so taller tiles would be bound by TMA issue);
// taller ones read rows the dispatch copied into expert order.
constexpr int kGatherMaxBn = 32;

struct Workspace {
  float* logits_part = nullptr;   // [splits][T][E]
  int32_t* ids = nullptr;         // [T][k]
  float* wts = nullptr;           // [T][k]
  int32_t* sched = nullptr;       // [64] unit counters of the pair GEMMs (zeroed per forward)
  int32_t* counts = nullptr;      // [E]            (zeroed per forward)
  uint32_t* bitmap = nullptr;     // [E][W] token bitmaps, W = ceil(Tmax/32) (zeroed per forward)
  int32_t* word_prefix = nullptr; // [E][W]
  int32_t* offsets = nullptr;     // [G+1] row offset of each group
  int32_t* unit_base = nullptr;   // [2][G+1] per-GEMM unit prefix
  int32_t* pair_row = nullptr;    // [T*k] row of each (token, slot)
  int32_t* row_token = nullptr;   // [Rmax] token of each row
  // B rows of the gate/up GEMM. Tall row tiles: [Rmax][d] gathered rows
  // (BF16, or e4m3 with scales xs [Rmax][d/128]) in row order. Short row
  // tiles gather from x itself; then, for FP8, rows [0, T) hold each
  // token's quantised x once (scales likewise).
  void* xp = nullptr;
  float* xs = nullptr;
  void* hbuf = nullptr;           // [Rmax][f] SwiGLU output, BF16 or e4m3
  float* hs = nullptr;            // [Rmax][f/128] FP8 scales of h
  uint16_t* out = nullptr;        // [Rmax][d] BF16 per-row expert outputs
  uint32_t* status = nullptr;     // device status word
  uint32_t* sync = nullptr;       // [2 + G] single-launch layer: grid barrier, abort, per-group
                                  // finished gate/up warps (zeroed per forward)
  void* x_stage[2] = {};          // [Tmax][d] BF16 staging of the host entry points, used in turn
  void* y_stage[2] = {};          // [Tmax][d]
  size_t zero_bytes = 0;          // bytes of the sched+counts+bitmap region cleared per forward
};

struct Weights {
  float* router = nullptr;  // [E][d]
  void* router_cat = nullptr;  // [E][3d] BF16: W_g = hi + mid + lo
  float* bias = nullptr;    // [E]
  void* gate = nullptr;     // [G][f][d]
  void* up = nullptr;       // [G][f][d]
  void* down = nullptr;     // [G][d][f]
  float* gate_s = nullptr;  // [G][f/128][d/128]
  float* up_s = nullptr;
  float* down_s = nullptr;  // [G][d/128][f/128]
  bool loaded = false;
};

}  // namespace smoe

struct moe_handle {
  moe_config_t cfg;
  int device = 0;
  int num_sms = 148;
  smoe::Dims dims{};
  smoe::Weights w;
  smoe::Workspace ws;
  // TMA descriptors: weights (one per projection); the gathered rows and h,
  // once per row-tile height 16 * (i + 1), i < 16; and tm_xg, the
  // one-row-box map short row tiles gather token rows through (over the
  // quantised rows [0, T) of xp for FP8, made once; over the caller's x for
  // BF16, made by each forward that gathers)
  CUtensorMap tm_gate, tm_up, tm_down, tm_router;
  CUtensorMap tm_xp[16], tm_h[16], tm_xg;
  int router_max_splits = 1;
  int64_t launches = 0;
  // options of the forward being launched: GEMM pipeline wait limit (0 =
  // default) and the test stall of the gate/up GEMM
  uint64_t fwd_wait_ns = 0;
  bool fwd_stall = false;
  std::string last_error;
  // per-phase profiling
  std::vector<cudaEvent_t> prof_events;
  int prof_cap = 0, prof_next = 0;
  // forwards run as one launch time their phases with device timestamps
  uint64_t* prof_stamps = nullptr;  // [prof_cap][MOE_NUM_PHASES + 1] globaltimer ns
  std::vector<char> prof_small;
  // host-memory entry points: upload and download streams, and per staging
  // buffer b the events "x uploaded", "forward done", "y downloaded"
  cudaStream_t up = nullptr, down = nullptr;
  cudaEvent_t ev_x[2] = {}, ev_fwd[2] = {}, ev_y[2] = {};
  uint64_t host_calls = 0;
  // forwards replayed as CUDA graphs, keyed by (T, x, y); captured and
  // replayed on `cap`, ordered against the caller's stream by ev_in / ev_out
  struct Graph {
    int64_t T = 0;
    const void* x = nullptr;
    void* y = nullptr;
    cudaGraphExec_t exec = nullptr;
    int64_t launches = 0;  // kernels in the graph
    uint64_t last_use = 0;
    bool failed = false;
  };
  Graph graphs[8];
  uint64_t graph_clock = 0;
  cudaStream_t cap = nullptr;
  cudaEvent_t ev_in = nullptr, ev_out = nullptr;
};

namespace smoe {

// router.cu
int router_splits(const Dims& dm, int64_t T, int num_sms);
cudaError_t launch_router_logits(moe_handle* h, const void* x, int T, int splits, cudaStream_t s);
cudaError_t launch_router_topk(moe_handle* h, int T, int splits, const int32_t* forced,
                               cudaStream_t s, int32_t* ids_out, float* wts_out,
                               float* logits_out);
cudaError_t launch_router_split(moe_handle* h, cudaStream_t s);
// gemm_promoted.cu: the router's logits on the tensor cores (T >= kTensorRouterMinT)
cudaError_t launch_router_gemm(moe_handle* h, const void* x, int T, cudaStream_t s);
constexpr int kTensorRouterMinT = 512;
constexpr int kTensorRouterSplits = 3;  // one K slice per BF16 part of the router weight
cudaError_t launch_router_raw(const void* x, const float* router_weight, const float* bias, int T,
                              int d, int E, int k, float scale, int norm, int splits, float* part,
                              int32_t* counts, uint32_t* bitmap, int W, uint32_t* status,
                              int32_t* ids, float* wts, cudaStream_t s);
// dispatch.cu
GemmPlan plan_gate_up(const Dims& dm, int64_t T);
GemmPlan plan_down(const Dims& dm, int64_t T);
cudaError_t launch_route_scan(moe_handle* h, int T, const GemmPlan& p1, const GemmPlan& p2,
                              cudaStream_t s);
cudaError_t launch_dispatch(moe_handle* h, const void* x, int T, bool gather, cudaStream_t s);
cudaError_t launch_combine(moe_handle* h, void* y, int T, cudaStream_t s);
cudaError_t launch_combine_rows(const void* pair_out, const float* wts, const void* shared, int T,
                                int d, int k, void* y, cudaStream_t s);
cudaError_t launch_act_quant(const void* x, int64_t rows, int d, uint8_t* q, float* s,
                             cudaStream_t st);
// layer_small.cu: the whole layer in one cooperative launch (16-row tiles)
bool small_layer_supported(const Dims& dm, int64_t T, int64_t max_t);
cudaError_t launch_small_layer(moe_handle* h, const void* x, int T, void* y,
                               const int32_t* forced, int32_t* ids_out, float* wts_out,
                               float* logits_out, uint64_t* stamps, cudaStream_t s);
// gemm_bf16.cu / gemm_promoted.cu
cudaError_t launch_gemm_bf16(moe_handle* h, bool gated, const GemmPlan& p, cudaStream_t s);
cudaError_t launch_gemm_bf16_pair(moe_handle* h, bool gated, const GemmPlan& p, cudaStream_t s);
bool pair_bn_supported(int bn);
cudaError_t launch_gemm_fp8(moe_handle* h, bool gated, const GemmPlan& p, cudaStream_t s);
int bn_index(int bn);
// api.cu
bool make_tmap(CUtensorMap* m, CUtensorMapDataType dt, int rank, void* base, const uint64_t* dims,
               const uint64_t* strides_bytes, const uint32_t* box, std::string* err);

}  // namespace smoe
