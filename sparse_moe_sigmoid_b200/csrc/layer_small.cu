// The whole layer in one launch for small batches (decode): router logits,
// noaux_tc top-k, scan, placement, gate/up GEMM + SwiGLU, down GEMM and the
// weighted combine with the shared expert, in one persistent kernel of one
// CTA per SM.
//
// Why: at decode sizes ("Behind Kimi-K2's Config" §2.1: decode is
// memory-bound and the batch is capped by the time between output tokens)
// the layer is seven short phases; as separate kernels each boundary costs a
// launch, a drain and a ramp-up, and the down projection cannot start before
// the last gate/up tile has finished. Here the phases run back to back
// inside one launch, separated by grid-wide barriers, and the two GEMMs form
// one pipeline: the units of every gate/up tile come first, then those of
// the down projection, and a down unit of expert g only waits (bounded) for
// a counter of g's finished gate/up tiles, so the down projection of early
// experts overlaps the gate/up tiles of later ones.
//
// The arithmetic is the phase kernels' (route_common.cuh for routing,
// placement, quantisation and the combine step; the same MMA shapes, SwiGLU
// and FP8 promotion as gemm_bf16.cu / gemm_promoted.cu with 16-row tiles),
// except the router logits, which sum each dot product in another order.
//
// Measured against the phase kernels on one B200: the routing phases are
// cheaper here, but the gate/up tiles stream 10-25% slower (decode T = 64:
// 3.62 vs 3.38 ms; FP8 T = 16: 1.02 vs 0.87 ms; FP8 T = 1: 0.127 vs
// 0.112 ms). It is therefore opt-in per handle (single_launch_max_tokens,
// default 0).
//
// Launch: cooperative (every CTA resident at once, or the launch fails), one
// CTA of six warps per SM: warp 0 loads (TMA), warp 1 owns TMEM and issues
// the MMAs, warps 2-5 drain the accumulators; all six take part in the
// CUDA-core phases. Every wait is bounded: a grid barrier, a readiness
// counter or a pipeline wait that runs out sets MOE_DEVICE_WAIT_TIMEOUT and a
// global abort word, and every CTA winds down (its loads land, TMEM is freed)
// and returns.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "gemm_common.cuh"
#include "internal.h"
#include "route_common.cuh"
#include "sm100.cuh"

namespace smoe {

using namespace sm100;

namespace {

constexpr int kBN = 16;            // rows per tile: the tile height of these batch sizes
constexpr int kThreads = 192;      // six warps
constexpr int kA = 128 * 128;      // one 128-row weight tile, 128 bytes of K per row
constexpr int kB = kBN * 128;      // the tile's 16 rows of B
constexpr int kStage = 2 * kA + kB;
constexpr int kStages = 6;
constexpr int kMaxKB = 128;        // K blocks of the longer GEMM (d / 64 for BF16)
constexpr int kTokChunk = 8;       // router: tokens per dot-product pass
static_assert(kStage % 1024 == 0, "stages keep 1024-byte alignment");

struct SmallArgs {
  const __nv_bfloat16* x;
  int T, d, f, E, k, ns, G;
  const float* router;
  const float* bias;
  float scale;
  int norm, n_group, topk_group;
  const int32_t* forced;
  float* logits;  // [T][E]
  int32_t* ids;
  float* wts;
  int32_t* counts;
  uint32_t* bitmap;
  int W;
  int32_t* word_prefix;
  int32_t* offsets;    // [G + 1]
  int32_t* unit_base;  // [2][G + 1]
  int32_t* pair_row;
  int32_t* row_token;
  uint8_t* xq;  // FP8: rows [0, T) hold each token's quantised x
  float* xs;
  void* h;      // [R][f] BF16 or e4m3
  float* hs;    // FP8: [R][f / 128]
  uint16_t* out;  // [R][d] BF16 per-row outputs
  __nv_bfloat16* y;
  const float* gate_s;
  const float* up_s;
  const float* down_s;
  int32_t* ids_out;
  float* wts_out;
  float* logits_out;
  uint32_t* status;
  uint32_t* sync;    // [0] grid barrier count, [1] abort, [2 + g] finished gate/up warps of g
  uint64_t* stamps;  // optional [8] phase boundaries (globaltimer ns)
  uint64_t wait_ns;
  int stall;
  int mt1, mt2;  // feature tiles per group: gate/up f / 128; down d / 256 (two halves per unit)
  int kb1, kb2;  // K blocks of gate/up and down
};

__device__ __forceinline__ uint32_t ld_acquire(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Generic-proxy global writes before, async-proxy (TMA) reads after.
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

__device__ __forceinline__ void stamp(const SmallArgs& a, int p) {
  if (a.stamps && blockIdx.x == 0 && threadIdx.x == 0) a.stamps[p] = globaltimer();
}

// Grid-wide barrier on a counter that only grows during the forward (each
// barrier waits for gridDim.x more arrivals). Bounded: returns false when the
// wait ran out (after setting the status bit and the abort word) or another
// CTA aborted.
__device__ bool grid_sync(const SmallArgs& a, uint32_t& target, volatile uint32_t* ok_s,
                          uint64_t lim) {
  __syncthreads();
  if (threadIdx.x == 0) {
    volatile uint32_t* abort_g = a.sync + 1;
    target += gridDim.x;
    bool ok = *abort_g == 0;
    if (ok) {
      __threadfence();
      atomicAdd(a.sync, 1u);
      const uint64_t t0 = globaltimer();
      for (uint32_t i = 0;; ++i) {
        if (ld_acquire(a.sync) >= target) break;
        if (*abort_g) {
          ok = false;
          break;
        }
        if ((i & 15u) == 15u && globaltimer() - t0 > lim) {
          atomicOr(a.status, MOE_DEVICE_WAIT_TIMEOUT);
          *abort_g = 1;
          ok = false;
          break;
        }
      }
    }
    *ok_s = ok ? 1u : 0u;
  }
  __syncthreads();
  return *ok_s != 0;
}

// Wait until group g's gate/up tiles are all stored (each of the four
// epilogue warps of every gate/up unit of g adds one). Bounded.
__device__ bool wait_ready(const SmallArgs& a, int g, uint32_t need, uint64_t lim) {
  volatile uint32_t* abort_g = a.sync + 1;
  const uint32_t* cnt = a.sync + 2 + g;
  const uint64_t t0 = globaltimer();
  for (uint32_t i = 0;; ++i) {
    if (ld_acquire(cnt) >= need) return true;
    if (*abort_g) return false;
    if ((i & 15u) == 15u && globaltimer() - t0 > lim) {
      atomicOr(a.status, MOE_DEVICE_WAIT_TIMEOUT);
      *abort_g = 1;
      return false;
    }
  }
}

// Router logits: CTAs split (8-token chunk) x (expert range); the chunk's x
// rows sit in shared memory. The six warps split K in six contiguous parts
// and each lane strides its part by 4 (float4 of the fp32 router row, exact
// BF16 products, fp32 sums), all of the CTA's experts at once so that their
// row loads are in flight together; the six partial sums of each (expert,
// token) are then added in warp order through shared memory.
constexpr int kRouterMaxE = 8;  // experts per CTA per pass
__device__ void phase_router(const SmallArgs& a, uint8_t* scratch) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nc = (a.T + kTokChunk - 1) / kTokChunk;
  const int nb = max(1, static_cast<int>(gridDim.x) / nc);
  if (static_cast<int>(blockIdx.x) >= nc * nb) return;
  const int chunk = blockIdx.x / nb, r = blockIdx.x % nb;
  const int t0 = chunk * kTokChunk, tn = min(kTokChunk, a.T - t0);
  const int e_lo = r * a.E / nb, e_hi = (r + 1) * a.E / nb;
  __nv_bfloat16* xs = reinterpret_cast<__nv_bfloat16*>(scratch);
  // partial sums [6 warps][kRouterMaxE][kTokChunk] after the x chunk
  float* red = reinterpret_cast<float*>(scratch + (size_t)kTokChunk * a.d * 2);
  const uint4* src = reinterpret_cast<const uint4*>(a.x + (size_t)t0 * a.d);
  uint4* dst = reinterpret_cast<uint4*>(xs);
  for (int i = threadIdx.x; i < tn * a.d / 8; i += kThreads) dst[i] = __ldg(src + i);
  __syncthreads();
  // this warp's K part: a multiple of 128 columns (a.d is a multiple of 256)
  const int part = ((a.d / 128 + 5) / 6) * 128;
  const int k_lo = warp * part, k_hi = min(a.d, k_lo + part);
  for (int eb = e_lo; eb < e_hi; eb += kRouterMaxE) {
    const int ne = min(kRouterMaxE, e_hi - eb);
    float acc[kRouterMaxE][kTokChunk];
#pragma unroll
    for (int q = 0; q < kRouterMaxE; ++q)
#pragma unroll
      for (int t = 0; t < kTokChunk; ++t) acc[q][t] = 0.f;
    for (int c = k_lo + lane * 4; c < k_hi; c += 128) {
      float4 wv[kRouterMaxE];
#pragma unroll
      for (int q = 0; q < kRouterMaxE; ++q)
        if (q < ne) wv[q] = __ldg(reinterpret_cast<const float4*>(a.router + (size_t)(eb + q) * a.d + c));
#pragma unroll
      for (int t = 0; t < kTokChunk; ++t) {
        if (t < tn) {
          const uint2 raw = *reinterpret_cast<const uint2*>(xs + (size_t)t * a.d + c);
          const float2 p = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.x));
          const float2 v = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.y));
#pragma unroll
          for (int q = 0; q < kRouterMaxE; ++q) {
            if (q < ne) {
              acc[q][t] = fmaf(p.x, wv[q].x, acc[q][t]);
              acc[q][t] = fmaf(p.y, wv[q].y, acc[q][t]);
              acc[q][t] = fmaf(v.x, wv[q].z, acc[q][t]);
              acc[q][t] = fmaf(v.y, wv[q].w, acc[q][t]);
            }
          }
        }
      }
    }
#pragma unroll
    for (int q = 0; q < kRouterMaxE; ++q) {
#pragma unroll
      for (int t = 0; t < kTokChunk; ++t) {
        float v = acc[q][t];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
        if (lane == 0) red[(warp * kRouterMaxE + q) * kTokChunk + t] = v;
      }
    }
    __syncthreads();
    if (threadIdx.x < ne * kTokChunk) {
      const int q = threadIdx.x / kTokChunk, t = threadIdx.x % kTokChunk;
      if (t < tn) {
        float v = 0.f;
        for (int w6 = 0; w6 < kThreads / 32; ++w6) v += red[(w6 * kRouterMaxE + q) * kTokChunk + t];
        a.logits[(size_t)(t0 + t) * a.E + eb + q] = v;
      }
    }
    __syncthreads();
  }
}

// Offsets, unit prefixes (CTA 0) and the experts' bitmap word prefixes (the
// other CTAs, one warp per expert).
__device__ void phase_scan(const SmallArgs& a) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (blockIdx.x == 0) {
    if (warp != 0) return;
    // each lane scans a contiguous segment of groups; lane sums are scanned
    // across the warp
    const int n = a.G;
    const int per = (n + 31) / 32;
    const int lo = min(n, lane * per), hi = min(n, lo + per);
    int s0 = 0, s1 = 0, s2 = 0;
    for (int g = lo; g < hi; ++g) {
      const int c = g < a.E ? a.counts[g] : a.T;
      s0 += c;
      s1 += a.mt1 * ((c + kBN - 1) / kBN);
      s2 += a.mt2 * ((c + kBN - 1) / kBN);
    }
    int p0 = s0, p1 = s1, p2 = s2;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int q0 = __shfl_up_sync(0xffffffffu, p0, off);
      const int q1 = __shfl_up_sync(0xffffffffu, p1, off);
      const int q2 = __shfl_up_sync(0xffffffffu, p2, off);
      if (lane >= off) {
        p0 += q0;
        p1 += q1;
        p2 += q2;
      }
    }
    int o0 = p0 - s0, o1 = p1 - s1, o2 = p2 - s2;  // exclusive
    for (int g = lo; g < hi; ++g) {
      a.offsets[g] = o0;
      a.unit_base[g] = o1;
      a.unit_base[a.G + 1 + g] = o2;
      const int c = g < a.E ? a.counts[g] : a.T;
      o0 += c;
      o1 += a.mt1 * ((c + kBN - 1) / kBN);
      o2 += a.mt2 * ((c + kBN - 1) / kBN);
    }
    if (lane == 31) {
      a.offsets[n] = p0;
      a.unit_base[n] = p1;
      a.unit_base[a.G + 1 + n] = p2;
    }
    return;
  }
  const int words = (a.T + 31) / 32;
  for (int e = (blockIdx.x - 1) * (kThreads / 32) + warp; e < a.E;
       e += (gridDim.x - 1) * (kThreads / 32)) {
    int run = 0;
    for (int w0 = 0; w0 < words; w0 += 32) {
      const int wd = w0 + lane;
      const int v = wd < words ? __popc(a.bitmap[(size_t)e * a.W + wd]) : 0;
      int incl = v;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int q = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += q;
      }
      if (wd < words) a.word_prefix[(size_t)e * a.W + wd] = run + incl - v;
      run += __shfl_sync(0xffffffffu, incl, 31);
    }
  }
}

// Placement of every (token, slot) pair and shared-group row; FP8: each
// token's x quantised once into rows [0, T) of xq.
template <bool FP8>
__device__ void phase_place(const SmallArgs& a) {
  const int items = a.T * (a.k + a.ns);
  const int tid = blockIdx.x * kThreads + threadIdx.x;
  for (int i = tid; i < items; i += gridDim.x * kThreads) {
    int t;
    const int row = place_row(i, a.T, a.k, a.E, a.ids, a.bitmap, a.word_prefix, a.offsets, a.W, &t);
    if (i < a.T * a.k) a.pair_row[i] = row;
    a.row_token[row] = t;
  }
  if (FP8) {
    // one warp per (token, pair of 128-column groups): a half-warp per group
    const int lane = threadIdx.x & 31;
    const int pairs = a.d / 256;
    for (int wi = tid >> 5; wi < a.T * pairs; wi += gridDim.x * (kThreads / 32)) {
      const int t = wi / pairs, c = (wi - t * pairs) * 256;
      quant_row_e4m3(a.x + (size_t)t * a.d + c, 256, a.xq + (size_t)t * a.d + c,
                     a.xs + (size_t)t * (a.d / 128) + c / 128, lane);
    }
    fence_proxy_async_global();  // the GEMM gathers xq with TMA
  }
}

// y[t] = sum_j w[t, j] * out[row(t, j)] + sum_s out[shared row(s, t)], fp32 in
// slot order, rounded once to BF16 (combine_kernel's arithmetic).
__device__ void phase_combine(const SmallArgs& a) {
  const int per_tok = a.d / 8;
  const int items = a.T * per_tok;
  for (int i = blockIdx.x * kThreads + threadIdx.x; i < items; i += gridDim.x * kThreads) {
    const int t = i / per_tok;
    const int c = (i - t * per_tok) * 8;
    float acc[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[j] = 0.f;
    for (int j = 0; j < a.k; ++j) {
      const int row = a.pair_row[(size_t)t * a.k + j];
      add_row8<false>(acc, a.out + (size_t)row * a.d + c, a.wts[(size_t)t * a.k + j]);
    }
    for (int s = 0; s < a.ns; ++s)
      add_row8<false>(acc, a.out + (size_t)(a.offsets[a.E + s] + t) * a.d + c, 1.f);
    uint32_t pk[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      __nv_bfloat162 b = __floats2bfloat162_rn(acc[2 * j], acc[2 * j + 1]);
      pk[j] = *reinterpret_cast<uint32_t*>(&b);
    }
    *reinterpret_cast<uint4*>(a.y + (size_t)t * a.d + c) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
  }
}

// A GEMM unit of the combined sequence: gate/up units of every group first
// (128 features, gate and up tiles), then the down units (256 output
// features as two 128-row tiles).
struct SmallUnit {
  bool gu;
  Unit un;
  int kb;
};

// The unit numbering of gemm_common.cuh (group, feature tile, row tile
// innermost), decoded with plain loads: the offsets and unit prefixes are
// written earlier in this launch, which the read-only path does not see.
__device__ __forceinline__ SmallUnit decode_small(const SmallArgs& a, int u, int U1) {
  SmallUnit s;
  s.gu = u < U1;
  const int32_t* ub = a.unit_base + (s.gu ? 0 : a.G + 1);
  const int local = s.gu ? u : u - U1;
  int lo = 0, hi = a.G;  // last group whose first unit is <= local
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (ub[mid] <= local) lo = mid;
    else hi = mid;
  }
  const int r0 = a.offsets[lo];
  const int cnt = a.offsets[lo + 1] - r0;
  const int nt = (cnt + kBN - 1) / kBN;
  const int rel = local - ub[lo];
  s.un.g = lo;
  s.un.mt = rel / nt;
  const int ti = rel - s.un.mt * nt;
  s.un.row0 = r0 + ti * kBN;
  s.un.nvalid = min(kBN, cnt - ti * kBN);
  s.un.split = 0;
  s.kb = s.gu ? a.kb1 : a.kb2;
  return s;
}

// gate/up tiles of group g: feature tiles x row tiles (its rows are offsets[g+1] - offsets[g])
__device__ __forceinline__ uint32_t ready_need(const SmallArgs& a, int g) {
  const int c = a.offsets[g + 1] - a.offsets[g];
  return 4u * static_cast<uint32_t>(a.mt1 * ((c + kBN - 1) / kBN));
}

template <bool FP8>
__global__ void __launch_bounds__(kThreads, 1)
    small_layer_kernel(const __grid_constant__ CUtensorMap tmG,
                       const __grid_constant__ CUtensorMap tmU,
                       const __grid_constant__ CUtensorMap tmD,
                       const __grid_constant__ CUtensorMap tmX,
                       const __grid_constant__ CUtensorMap tmH, const SmallArgs a) {
  constexpr int kK = FP8 ? 128 : 64;  // K elements per stage (128 bytes)
  // TMEM: BF16 double-buffered accumulators of 2 x 16 columns; FP8 four
  // partial buffers of 2 x 16 columns
  constexpr int kBufs = FP8 ? 4 : 2;
  constexpr int kTmemCols = 128;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  float* sa_s = reinterpret_cast<float*>(smem + kStages * kStage);  // [kMaxKB][16] (FP8)
  float* sw_s = sa_s + kMaxKB * kBN;                                // [2][kMaxKB]
  float* amax_s = sw_s + 2 * kMaxKB;                                // [4][16]
  uint64_t* full = reinterpret_cast<uint64_t*>(amax_s + 4 * kBN);
  uint64_t* empty = full + kStages;
  uint64_t* tfull = empty + kStages;  // pfull for FP8
  uint64_t* tempty = tfull + 4;       // pempty for FP8
  uint64_t* drain = tempty + 4;
  uint64_t* grp = drain + 1;
  uint64_t* stallbar = grp + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(stallbar + 1);
  volatile uint32_t* abort_flag = tmem_slot + 1;
  volatile uint32_t* consumed = tmem_slot + 2;
  volatile uint32_t* issued = tmem_slot + 3;
  volatile uint32_t* ok_s = tmem_slot + 4;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint64_t lim = a.wait_ns ? a.wait_ns : kTimeoutNs;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 4; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 4);
    }
    mbar_init(drain, 1);
    mbar_init(grp, 128);
    mbar_init(stallbar, 1);
    *abort_flag = 0;
    *consumed = 0;
    *issued = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmG);
    tma_prefetch_desc(&tmU);
    tma_prefetch_desc(&tmD);
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmH);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  uint32_t target = 0;
  stamp(a, 0);

  // ---------------------------------------------------------- routing
  phase_router(a, smem);
  bool ok = grid_sync(a, target, ok_s, lim);
  stamp(a, 1);
  if (ok) {
    const TopkArgs ta{a.logits, 1, a.bias, a.T, a.E, a.k, a.scale, a.norm, a.forced, a.ids,
                      a.wts, a.counts, a.bitmap, a.W, a.status, a.ids_out, a.wts_out,
                      a.logits_out, a.n_group, a.topk_group};
    float* row = reinterpret_cast<float*>(smem) + warp * kMaxExperts;
    for (int t = blockIdx.x * (kThreads / 32) + warp; t < a.T; t += gridDim.x * (kThreads / 32))
      route_token(ta, t, row, lane);
    ok = grid_sync(a, target, ok_s, lim);
  }
  stamp(a, 2);
  if (ok) {
    phase_scan(a);
    ok = grid_sync(a, target, ok_s, lim);
  }
  stamp(a, 3);
  if (ok) {
    phase_place<FP8>(a);
    ok = grid_sync(a, target, ok_s, lim);
  }
  stamp(a, 4);

  // ------------------------------------------------------------- GEMMs
  const int U1 = ok ? a.unit_base[a.G] : 0;  // written in this launch: plain loads
  const int U = ok ? U1 + a.unit_base[a.G + 1 + a.G] : 0;
  const int ldh = a.f;
  // the routing phases used the ring's shared memory through the generic
  // proxy; TMA (async proxy) writes it from here on
  fence_proxy_async_smem();
  if (warp == 0) {
    if (ok) fence_proxy_async_global();  // xq / x rows and, later, h are read by TMA
    uint32_t it = 0;
    bool run = true;
    for (int u = blockIdx.x; u < U && run; u += gridDim.x) {
      // every gate/up unit precedes every down unit: from the first down
      // unit on, lane 0 streams alone (box loads need no other lane, and a
      // warp-wide loop with a shuffle and a warp barrier per stage measured
      // slower for box loads)
      if (u >= U1 && lane != 0) break;
      const SmallUnit su = decode_small(a, u, U1);
      int tok[4] = {};
      if (su.gu && 4 * lane < kBN) {
        // token rows of B (rows past the tile's valid ones repeat its first row)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int r = 4 * lane + j;
          tok[j] = a.row_token[su.un.row0 + (r < su.un.nvalid ? r : 0)];
        }
      }
      if (!su.gu) {  // lane 0 alone: h rows of this group must all be stored first
        run = wait_ready(a, su.un.g, ready_need(a, su.un.g), lim);
        if (!run) break;
        fence_proxy_async_global();
        for (int kb = 0; kb < su.kb; ++kb, ++it) {
          const int s = it % kStages;
          const uint32_t ph = (it / kStages) & 1u;
          if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag, lim)) {
            run = false;
            break;
          }
          uint8_t* st = smem + s * kStage;
          mbar_arrive_expect_tx(&full[s], kStage);
          tma_load_3d(st, &tmD, &full[s], kb * kK, su.un.mt * 256, su.un.g);
          tma_load_3d(st + kA, &tmD, &full[s], kb * kK, su.un.mt * 256 + 128, su.un.g);
          tma_load_2d(st + 2 * kA, &tmH, &full[s], kb * kK, su.un.row0);
          *issued = it + 1;
        }
        continue;
      }
      for (int kb = 0; kb < su.kb; ++kb, ++it) {
        const int s = it % kStages;
        const uint32_t ph = (it / kStages) & 1u;
        if (lane == 0) run = mbar_wait(&empty[s], ph ^ 1u, abort_flag, lim);
        run = __shfl_sync(0xffffffffu, run, 0);
        if (!run) break;
        uint8_t* st = smem + s * kStage;
        if (lane == 0) {
          mbar_arrive_expect_tx(&full[s], kStage);
          tma_load_3d(st, &tmG, &full[s], kb * kK, su.un.mt * 128, su.un.g);
          tma_load_3d(st + kA, &tmU, &full[s], kb * kK, su.un.mt * 128, su.un.g);
        }
        if (4 * lane < kBN)
          tma_gather4(st + 2 * kA + 4 * lane * 128, &tmX, &full[s], kb * kK, tok[0], tok[1],
                      tok[2], tok[3]);
        __syncwarp();
        if (lane == 0) *issued = it + 1;
      }
    }
    if (!run && lane == 0) {
      *abort_flag = 1;
      atomicOr(a.status, MOE_DEVICE_WAIT_TIMEOUT);
      *(a.sync + 1) = 1;
    }
  } else if (warp == 1) {
    if (lane == 0) {
      uint32_t it = 0, pit = 0;
      bool run = U > 0 && (!a.stall || mbar_wait(stallbar, 0, abort_flag, lim));
      int i = 0;
      const uint32_t idesc = make_idesc(FP8 ? 0u : 1u, kBN);
      for (int u = blockIdx.x; u < U && run; u += gridDim.x, ++i) {
        const SmallUnit su = decode_small(a, u, U1);
        if (!FP8) {
          const int acc = i % kBufs;
          if (!mbar_wait(&tempty[acc], ((i / kBufs) & 1) ^ 1, abort_flag, lim)) {
            run = false;
            break;
          }
          tc_fence_after();
        }
        for (int kb = 0; kb < su.kb; ++kb, ++it) {
          const int s = it % kStages;
          const uint32_t ph = (it / kStages) & 1u;
          const int pb = FP8 ? static_cast<int>(pit % kBufs) : i % kBufs;
          if ((FP8 && !mbar_wait(&tempty[pb], ((pit / kBufs) & 1u) ^ 1u, abort_flag, lim)) ||
              !mbar_wait(&full[s], ph, abort_flag, lim)) {
            run = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(smem + s * kStage);
          const uint64_t ad0 = sw128_kmajor_desc(a0);
          const uint64_t ad1 = sw128_kmajor_desc(a0 + kA);
          const uint64_t bd = sw128_kmajor_desc(a0 + 2 * kA);
          const uint32_t d0 = tmem_base + pb * 2 * kBN;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            // FP8: each block's partial starts fresh; BF16: the unit accumulates
            const uint32_t accum = FP8 ? (k ? 1u : 0u) : ((kb | k) ? 1u : 0u);
            if (FP8) {
              mma_fp8(d0, ad0 + 2 * k, bd + 2 * k, idesc, accum);
              mma_fp8(d0 + kBN, ad1 + 2 * k, bd + 2 * k, idesc, accum);
            } else {
              mma_bf16(d0, ad0 + 2 * k, bd + 2 * k, idesc, accum);
              mma_bf16(d0 + kBN, ad1 + 2 * k, bd + 2 * k, idesc, accum);
            }
          }
          mma_commit(&empty[s]);
          if (FP8) {
            mma_commit(&tfull[pb]);
            ++pit;
          }
          *consumed = it + 1;
        }
        if (!run) break;
        if (!FP8) mma_commit(&tfull[i % kBufs]);
      }
      if (!run && U > 0) {
        *abort_flag = 1;
        atomicOr(a.status, MOE_DEVICE_WAIT_TIMEOUT);
        *(a.sync + 1) = 1;
      }
      mma_commit(drain);
      mbar_wait(drain, 0, nullptr);
    }
  } else {
    // warps 2..5: drain (BF16) or promote (FP8) the accumulators of TMEM
    // lane quarter q; store h (gate/up) or the per-row outputs (down)
    const int q = warp & 3;
    const int ptid = threadIdx.x - 64;
    const uint32_t tq = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    uint32_t pit = 0, gph = 0;
    bool run = true;
    auto group_sync = [&]() {
      mbar_arrive(grp);
      const bool r = mbar_wait(grp, gph, abort_flag, lim);
      gph ^= 1u;
      return r;
    };
    int i = 0;
    for (int u = blockIdx.x; u < U && run; u += gridDim.x, ++i) {
      const SmallUnit su = decode_small(a, u, U1);
      const Unit& un = su.un;
      float acc0[kBN], acc1[kBN];
      if (FP8) {
        // this tile's activation and weight block scales
        if (!su.gu && ptid == 0)  // the h scales of the group must be stored
          *ok_s = wait_ready(a, un.g, ready_need(a, un.g), lim) ? 1u : 0u;
        if (!group_sync()) {
          run = false;
          break;
        }
        if (!su.gu && *ok_s == 0) {
          run = false;
          break;
        }
        const int KB = su.kb;
        for (int e = ptid; e < KB * kBN; e += 128) {
          const int kb = e / kBN, j = e - kb * kBN;
          float v = 0.f;
          if (j < un.nvalid) {
            v = su.gu ? a.xs[(size_t)a.row_token[un.row0 + j] * KB + kb]
                      : a.hs[(size_t)(un.row0 + j) * KB + kb];
          }
          sa_s[e] = v;
        }
        for (int e = ptid; e < KB; e += 128) {
          if (su.gu) {
            const size_t r0 = ((size_t)un.g * a.mt1 + un.mt) * KB;
            sw_s[e] = __ldg(a.gate_s + r0 + e);
            sw_s[kMaxKB + e] = __ldg(a.up_s + r0 + e);
          } else {
            const size_t r0 = ((size_t)un.g * 2 * a.mt2 + 2 * un.mt) * KB;
            sw_s[e] = __ldg(a.down_s + r0 + e);
            sw_s[kMaxKB + e] = __ldg(a.down_s + r0 + KB + e);
          }
        }
        if (!group_sync()) {
          run = false;
          break;
        }
#pragma unroll
        for (int j = 0; j < kBN; ++j) {
          acc0[j] = 0.f;
          acc1[j] = 0.f;
        }
        for (int kb = 0; kb < KB; ++kb, ++pit) {
          const int pb = pit % kBufs;
          if (!mbar_wait(&tfull[pb], (pit / kBufs) & 1u, abort_flag, lim)) {
            run = false;
            break;
          }
          tc_fence_after();
          uint32_t g[16], v[16];
          tmem_ld16(tq + pb * 2 * kBN, g);
          tmem_ld16(tq + pb * 2 * kBN + kBN, v);
          tmem_ld_wait();
          const float sw0 = sw_s[kb], sw1 = sw_s[kMaxKB + kb];
#pragma unroll
          for (int j = 0; j < kBN; ++j) {
            const float sx = sa_s[kb * kBN + j];
            acc0[j] = fmaf(__uint_as_float(g[j]), sw0 * sx, acc0[j]);
            acc1[j] = fmaf(__uint_as_float(v[j]), sw1 * sx, acc1[j]);
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&tempty[pb]);
        }
        if (!run) break;
      } else {
        const int acc = i % kBufs;
        if (!mbar_wait(&tfull[acc], (i / kBufs) & 1, abort_flag, lim)) {
          run = false;
          break;
        }
        tc_fence_after();
        uint32_t g[16], v[16];
        tmem_ld16(tq + acc * 2 * kBN, g);
        tmem_ld16(tq + acc * 2 * kBN + kBN, v);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < kBN; ++j) {
          acc0[j] = __uint_as_float(g[j]);
          acc1[j] = __uint_as_float(v[j]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[acc]);
      }

      if (su.gu) {
        const int feat = un.mt * 128 + q * 32 + lane;
        // h = silu(g) * u (IEEE expf and division, as the other GEMM kernels)
#pragma unroll
        for (int j = 0; j < kBN; ++j) acc0[j] = acc0[j] / (1.f + expf(-acc0[j])) * acc1[j];
        if (FP8) {
          // per-row e4m3 quantisation over this tile's 128 features
#pragma unroll
          for (int j = 0; j < kBN; ++j) {
            const uint32_t m = __reduce_max_sync(0xffffffffu, __float_as_uint(fabsf(acc0[j])));
            if (lane == 0) amax_s[q * kBN + j] = __uint_as_float(m);
          }
          if (!group_sync()) {
            run = false;
            break;
          }
          uint8_t* hq = static_cast<uint8_t*>(a.h);
#pragma unroll
          for (int j = 0; j < kBN; ++j) {
            if (j < un.nvalid) {
              const float amax = fmaxf(fmaxf(amax_s[j], amax_s[kBN + j]),
                                       fmaxf(amax_s[2 * kBN + j], amax_s[3 * kBN + j]));
              const float sh = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
              const size_t row = static_cast<size_t>(un.row0 + j);
              float2 pr;
              pr.x = __fdiv_rn(acc0[j], sh);
              pr.y = 0.f;
              const __nv_fp8x2_storage_t b =
                  __nv_cvt_float2_to_fp8x2(pr, __NV_SATFINITE, __NV_E4M3);
              hq[row * ldh + feat] = static_cast<uint8_t>(b & 0xFF);
              if (q == 0 && lane == 0) a.hs[row * a.mt1 + un.mt] = sh;
            }
          }
        } else {
          __nv_bfloat16* hb = static_cast<__nv_bfloat16*>(a.h);
#pragma unroll
          for (int j = 0; j < kBN; ++j)
            if (j < un.nvalid) hb[(size_t)(un.row0 + j) * ldh + feat] = __float2bfloat16_rn(acc0[j]);
        }
        // publish h (read by TMA) and its scales (generic loads) of this tile:
        // every lane orders its stores for the async proxy, then one lane
        // releases them gpu-wide with the counter
        fence_proxy_async_global();
        __syncwarp();
        if (lane == 0) {
          __threadfence();
          atomicAdd(a.sync + 2 + un.g, 1u);
        }
      } else {
        const int feat = un.mt * 256 + q * 32 + lane;
        __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(a.out);
#pragma unroll
        for (int j = 0; j < kBN; ++j) {
          if (j < un.nvalid) {
            const size_t row = static_cast<size_t>(un.row0 + j);
            o[row * a.d + feat] = __float2bfloat16_rn(acc0[j]);
            o[row * a.d + feat + 128] = __float2bfloat16_rn(acc1[j]);
          }
        }
      }
    }
    if (!run && lane == 0) {
      *abort_flag = 1;
      atomicOr(a.status, MOE_DEVICE_WAIT_TIMEOUT);
      *(a.sync + 1) = 1;
    }
  }

  // wind-down of the GEMM pipeline: loads issued but never consumed land
  // before the CTA moves on
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (*abort_flag && warp == 0 && lane == 0) {
    for (uint32_t j = *consumed; j < *issued; ++j)
      mbar_wait(&full[j % kStages], (j / kStages) & 1u, nullptr);
  }
  ok = ok && !*abort_flag && grid_sync(a, target, ok_s, lim);
  if (a.stamps && blockIdx.x == 0 && threadIdx.x == 0) {
    // both GEMMs ran in one pipeline: the down phase is reported empty
    const uint64_t t = globaltimer();
    a.stamps[5] = t;
    a.stamps[6] = t;
  }
  if (ok) phase_combine(a);
  __syncthreads();
  stamp(a, 7);
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, kTmemCols);
}

constexpr int kSmallSmem = 1024 + kStages * kStage + (kMaxKB * kBN + 2 * kMaxKB + 4 * kBN) * 4 +
                           (2 * kStages + 4 + 4 + 3) * 8 + 32;

}  // namespace

bool small_layer_supported(const Dims& dm, int64_t T, int64_t max_t) {
  if (dm.E == 0 || T < 1 || T > kSmallMaxT || T > max_t) return false;
  const GemmPlan p1 = plan_gate_up(dm, T), p2 = plan_down(dm, T);
  if (p1.bn != kBN || p2.bn != kBN || p1.pair || p2.pair) return false;
  if (dm.d % 256 || dm.f % 128) return false;
  const int kb1 = dm.fp8 ? dm.d / 128 : dm.d / 64;
  const int kb2 = dm.fp8 ? dm.f / 128 : dm.f / 64;
  if (kb1 > kMaxKB || kb2 > kMaxKB) return false;
  // the router's x chunk must fit the shared-memory ring
  if (static_cast<size_t>(kTokChunk) * dm.d * 2 + 6 * kRouterMaxE * kTokChunk * 4 >
      static_cast<size_t>(kStages) * kStage)
    return false;
  return true;
}

cudaError_t launch_small_layer(moe_handle* h, const void* x, int T, void* y,
                               const int32_t* forced, int32_t* ids_out, float* wts_out,
                               float* logits_out, uint64_t* stamps, cudaStream_t s) {
  const Dims& dm = h->dims;
  SmallArgs a{};
  a.x = static_cast<const __nv_bfloat16*>(x);
  a.T = T;
  a.d = dm.d;
  a.f = dm.f;
  a.E = dm.E;
  a.k = dm.k;
  a.ns = dm.ns;
  a.G = dm.G;
  a.router = h->w.router;
  a.bias = h->w.bias;
  a.scale = h->cfg.routed_scaling_factor;
  a.norm = h->cfg.norm_topk_prob;
  a.n_group = h->cfg.n_group;
  a.topk_group = h->cfg.topk_group;
  a.forced = forced;
  a.logits = h->ws.logits_part;
  a.ids = h->ws.ids;
  a.wts = h->ws.wts;
  a.counts = h->ws.counts;
  a.bitmap = h->ws.bitmap;
  a.W = static_cast<int>((dm.Tmax + 31) / 32);
  a.word_prefix = h->ws.word_prefix;
  a.offsets = h->ws.offsets;
  a.unit_base = h->ws.unit_base;
  a.pair_row = h->ws.pair_row;
  a.row_token = h->ws.row_token;
  a.xq = static_cast<uint8_t*>(h->ws.xp);
  a.xs = h->ws.xs;
  a.h = h->ws.hbuf;
  a.hs = h->ws.hs;
  a.out = h->ws.out;
  a.y = static_cast<__nv_bfloat16*>(y);
  a.gate_s = h->w.gate_s;
  a.up_s = h->w.up_s;
  a.down_s = h->w.down_s;
  a.ids_out = ids_out;
  a.wts_out = wts_out;
  a.logits_out = logits_out;
  a.status = h->ws.status;
  a.sync = h->ws.sync;
  a.stamps = stamps;
  a.wait_ns = h->fwd_wait_ns;
  a.stall = h->fwd_stall ? 1 : 0;
  a.mt1 = dm.f / 128;
  a.mt2 = dm.d / 256;
  a.kb1 = dm.fp8 ? dm.d / 128 : dm.d / 64;
  a.kb2 = dm.fp8 ? dm.f / 128 : dm.f / 64;

  // tm_xg: over the quantised token rows (FP8, made at create), or over the
  // caller's x (BF16, made by the forward)
  const CUtensorMap& tmx = h->tm_xg;
  auto kern = dm.fp8 ? small_layer_kernel<true> : small_layer_kernel<false>;
  static bool configured[2][64] = {};
  if (h->device < 64 && !configured[dm.fp8][h->device]) {
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmallSmem);
    if (e != cudaSuccess) return e;
    configured[dm.fp8][h->device] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(h->num_sms));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmallSmem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, h->tm_gate, h->tm_up, h->tm_down, tmx,
                                     h->tm_h[0], a);
  h->launches++;
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace smoe
