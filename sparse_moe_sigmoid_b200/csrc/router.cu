// Router of the K2 MoE layer: logits, sigmoid scores, noaux_tc biased top-k,
// normalisation and routed scaling.
//
// Config fields (scoring_func sigmoid, topk_method noaux_tc, n_group 1,
// num_experts_per_tok 8, norm_topk_prob true, routed_scaling_factor 2.827):
// "Kimi K2 Base" / "Kimi K2 0905" model cards, raw config field tables.
//
// Kernel 1 (router_logits_kernel): logits = x . W_g^T in fp32 on CUDA cores.
//   The router weight is fp32, and tensor-core TF32 would move logits by
//   ~1e-3, enough to change which experts win; so this is an exact-product
//   fp32 FMA GEMM tiled 64 tokens x 64 experts. Small T splits the hidden
//   dimension into `splits` slices so the grid covers the SMs; the partial
//   sums land in [splits][T][E] and are added in slice order by kernel 2,
//   which keeps the result deterministic.
// Kernel 2 (router_topk_kernel): one warp per token. Lane l holds experts
//   l, l+32, ...; it adds the partials, takes the sigmoid, forms the key
//   score + bias, applies the group filter when n_group > 1 (below), and the
//   warp extracts the k largest keys (ties to the lower expert index) by k
//   rounds of a shuffle arg-max. The weights use the
//   unbiased scores: w = score / sum(selected scores) * 2.827. It also counts
//   tokens per expert and sets the token's bit in the expert's bitmap, which
//   the dispatch uses to place each (token, slot) pair.
#include <cuda_bf16.h>
#include <math.h>

#include "internal.h"
#include "route_common.cuh"

namespace smoe {

int router_splits(const Dims& dm, int64_t T, int num_sms) {
  const int64_t tiles = ((dm.E + kRouterTile - 1) / kRouterTile) *
                        ((T + kRouterTile - 1) / kRouterTile);
  int64_t want = (2 * num_sms + tiles - 1) / tiles;
  // the top-k kernel adds the slices serially per lane: keep them few
  int64_t max_splits = dm.d / kRouterKTile < kRouterMaxSplits ? dm.d / kRouterKTile
                                                               : kRouterMaxSplits;
  if (want < 1) want = 1;
  if (want > max_splits) want = max_splits;
  // each slice is a multiple of the 32-wide K tile
  int64_t kps = (dm.d + want - 1) / want;
  kps = (kps + kRouterKTile - 1) / kRouterKTile * kRouterKTile;
  return static_cast<int>((dm.d + kps - 1) / kps);
}

static int router_kps(const Dims& dm, int splits) {
  int kps = (dm.d + splits - 1) / splits;
  return (kps + kRouterKTile - 1) / kRouterKTile * kRouterKTile;
}

__global__ void __launch_bounds__(256) router_logits_kernel(const __nv_bfloat16* __restrict__ x,
                                                            const float* __restrict__ W,
                                                            float* __restrict__ part, int T,
                                                            int E, int d, int kps) {
  __shared__ __align__(16) float Xs[kRouterKTile][kRouterTile + 4];
  __shared__ __align__(16) float Ws[kRouterKTile][kRouterTile + 4];
  const int e0 = blockIdx.x * kRouterTile;
  const int t0 = blockIdx.y * kRouterTile;
  const int split = blockIdx.z;
  const int kbeg = split * kps;
  const int kend = min(d, kbeg + kps);
  const int tid = threadIdx.x;
  const int ty = tid >> 4, tx = tid & 15;
  const int lr = tid >> 2, lc = (tid & 3) * 8;  // loader: row, 8-wide column group

  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;

  // global loads of K tile k0 + kRouterKTile are issued before tile k0 is
  // multiplied (register double buffering: the loop is latency-bound at the
  // small T this kernel serves)
  const bool t_ok = t0 + lr < T, e_ok = e0 + lr < E;
  const __nv_bfloat16* xrow = x + (size_t)(t0 + lr) * d + lc;
  const float* wrow = W + (size_t)(e0 + lr) * d + lc;
  uint4 xr = make_uint4(0u, 0u, 0u, 0u);
  float4 wa = make_float4(0.f, 0.f, 0.f, 0.f), wb = wa;
  if (kbeg < kend) {
    if (t_ok) xr = *reinterpret_cast<const uint4*>(xrow + kbeg);
    if (e_ok) {
      wa = *reinterpret_cast<const float4*>(wrow + kbeg);
      wb = *reinterpret_cast<const float4*>(wrow + kbeg + 4);
    }
  }
  for (int k0 = kbeg; k0 < kend; k0 += kRouterKTile) {
    {
      const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&xr);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f2 = __bfloat1622float2(p[i]);
        Xs[lc + 2 * i][lr] = f2.x;
        Xs[lc + 2 * i + 1][lr] = f2.y;
      }
      Ws[lc + 0][lr] = wa.x; Ws[lc + 1][lr] = wa.y; Ws[lc + 2][lr] = wa.z; Ws[lc + 3][lr] = wa.w;
      Ws[lc + 4][lr] = wb.x; Ws[lc + 5][lr] = wb.y; Ws[lc + 6][lr] = wb.z; Ws[lc + 7][lr] = wb.w;
    }
    __syncthreads();
    const int kn = k0 + kRouterKTile;
    if (kn < kend) {
      if (t_ok) xr = *reinterpret_cast<const uint4*>(xrow + kn);
      if (e_ok) {
        wa = *reinterpret_cast<const float4*>(wrow + kn);
        wb = *reinterpret_cast<const float4*>(wrow + kn + 4);
      }
    }
#pragma unroll
    for (int kk = 0; kk < kRouterKTile; ++kk) {
      const float4 a = *reinterpret_cast<const float4*>(&Xs[kk][ty * 4]);
      const float4 b = *reinterpret_cast<const float4*>(&Ws[kk][tx * 4]);
      const float av[4] = {a.x, a.y, a.z, a.w};
      const float bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int t = t0 + ty * 4 + i;
    if (t >= T) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int e = e0 + tx * 4 + j;
      if (e < E) part[((size_t)split * T + t) * E + e] = acc[i][j];
    }
  }
}

__global__ void __launch_bounds__(256) router_topk_kernel(TopkArgs a) {
  __shared__ float group_rows[256 / 32][kMaxExperts];  // one key row per warp (group filter)
  const int lane = threadIdx.x & 31;
  const int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (t >= a.T) return;
  route_token(a, t, group_rows[threadIdx.x >> 5], lane);
}

// Few tokens: one warp's k rounds over all E experts are a long serial chain
// (~2800 instructions for K2's E = 384, k = 8, one token measured at ~14 us).
// Here four warps share a token (a 128-thread group, two tokens per CTA):
// warp w takes the contiguous experts [w * chunk, (w + 1) * chunk), chunk =
// ceil(E / 4) <= 128, four per lane; it adds their partial logits in slice
// order and forms scores and keys exactly as route_token, then extracts its
// own k best (key descending, the lower expert first on equal keys) into
// shared memory; warp 0 of the group extracts the k best of those 4k
// candidates the same way and finishes as route_token does. The k best of all
// experts are among the candidates and the order is total, so the experts,
// their order, the weights and the bookkeeping are route_token's bit for bit.
// A token with a NaN key goes to route_token (its fallback for keys that
// compare false needs every expert). Unforced routing with n_group = 1 only.
constexpr int kSmallTopkWarps = 4;
constexpr int kSmallTopkPerLane = kMaxExperts / 32 / kSmallTopkWarps;
constexpr int kSmallTopkMaxT = 256;

__global__ void __launch_bounds__(256) router_topk_small_kernel(TopkArgs a) {
  constexpr int kC = kSmallTopkWarps * kMaxTopK;  // candidates per token, at most
  __shared__ float c_key[2][kC], c_sc[2][kC];
  __shared__ int c_id[2][kC];
  __shared__ int c_nan[2];
  const unsigned full = 0xffffffffu;
  const int g = threadIdx.x >> 7;        // token slot of this CTA
  const int w = (threadIdx.x >> 5) & 3;  // warp within the token's group
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * 2 + g;
  const bool live = t < a.T;
  const int E = a.E, k = a.k;
  const int chunk = (E + kSmallTopkWarps - 1) / kSmallTopkWarps;
  const int e0 = w * chunk;
  const int e1 = E < e0 + chunk ? E : e0 + chunk;
  if (threadIdx.x < 2) c_nan[threadIdx.x] = 0;
  __syncthreads();

  float key[kSmallTopkPerLane], sc[kSmallTopkPerLane];
  bool nan = false;
#pragma unroll
  for (int i = 0; i < kSmallTopkPerLane; ++i) {
    key[i] = -INFINITY;
    sc[i] = 0.f;
  }
  if (live) {
    float lg[kSmallTopkPerLane];
#pragma unroll
    for (int i = 0; i < kSmallTopkPerLane; ++i) lg[i] = 0.f;
#pragma unroll 4
    for (int s = 0; s < a.splits; ++s) {
      const float* ps = a.part + ((size_t)s * a.T + t) * E;
      float v[kSmallTopkPerLane];
#pragma unroll
      for (int i = 0; i < kSmallTopkPerLane; ++i) {
        const int e = e0 + lane + 32 * i;
        v[i] = e < e1 ? ps[e] : 0.f;
      }
#pragma unroll
      for (int i = 0; i < kSmallTopkPerLane; ++i) lg[i] += v[i];
    }
#pragma unroll
    for (int i = 0; i < kSmallTopkPerLane; ++i) {
      const int e = e0 + lane + 32 * i;
      if (e < e1) {
        const float l = lg[i];
        if (a.logits_out) a.logits_out[(size_t)t * E + e] = l;
        const float p = 1.f / (1.f + expf(-l));
        sc[i] = p;
        key[i] = p + a.bias[e];
        nan |= key[i] != key[i];
      }
    }
  }
  if (__any_sync(full, nan) && lane == 0) c_nan[g] = 1;

  // this warp's k best: round j's winner is kept by lane j
  float my_key = -INFINITY, my_sc = 0.f;
  int my_id = 0x7fffffff;
  uint32_t taken = 0;
  for (int j = 0; j < k; ++j) {
    float bk = -INFINITY;
    int bi = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < kSmallTopkPerLane; ++i) {
      const int e = e0 + lane + 32 * i;
      if (e < e1 && !((taken >> i) & 1u) && (key[i] > bk || (key[i] == bk && e < bi))) {
        bk = key[i];
        bi = e;
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float ok = __shfl_xor_sync(full, bk, off);
      const int oi = __shfl_xor_sync(full, bi, off);
      if (ok > bk || (ok == bk && oi < bi)) {
        bk = ok;
        bi = oi;
      }
    }
    float v = 0.f;
    if (bi < e1) {  // a winner (else no expert of this warp is left)
      const int r = bi - e0;
      if ((r & 31) == lane) taken |= 1u << (r >> 5);
#pragma unroll
      for (int i = 0; i < kSmallTopkPerLane; ++i)
        if (i == (r >> 5)) v = sc[i];
      v = __shfl_sync(full, v, r & 31);
    }
    if (lane == j) {
      my_key = bk;
      my_id = bi;
      my_sc = v;
    }
  }
  if (lane < k) {
    c_key[g][w * k + lane] = my_key;
    c_sc[g][w * k + lane] = my_sc;
    c_id[g][w * k + lane] = my_id;
  }
  __syncthreads();
  if (w != 0 || !live) return;
  if (c_nan[g]) {  // NaN keys: the one-warp routine and its fallback
    route_token(a, t, &c_key[g][0], lane);
    return;
  }

  // the k best of the 4k candidates (candidate c on lane c % 32, slot c / 32)
  const int nc = kSmallTopkWarps * k;
  float ck[kSmallTopkWarps], cs[kSmallTopkWarps];
  int ci[kSmallTopkWarps];
#pragma unroll
  for (int i = 0; i < kSmallTopkWarps; ++i) {
    const int c = lane + 32 * i;
    ck[i] = c < nc ? c_key[g][c] : -INFINITY;
    cs[i] = c < nc ? c_sc[g][c] : 0.f;
    ci[i] = c < nc ? c_id[g][c] : 0x7fffffff;
  }
  my_sc = 0.f;
  my_id = 0;
  taken = 0;
  for (int j = 0; j < k; ++j) {
    float bk = -INFINITY;
    int bi = 0x7fffffff, bc = 0;
#pragma unroll
    for (int i = 0; i < kSmallTopkWarps; ++i) {
      if (!((taken >> i) & 1u) && (ck[i] > bk || (ck[i] == bk && ci[i] < bi))) {
        bk = ck[i];
        bi = ci[i];
        bc = lane + 32 * i;
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float ok = __shfl_xor_sync(full, bk, off);
      const int oi = __shfl_xor_sync(full, bi, off);
      const int oc = __shfl_xor_sync(full, bc, off);
      if (ok > bk || (ok == bk && oi < bi)) {
        bk = ok;
        bi = oi;
        bc = oc;
      }
    }
    if ((bc & 31) == lane) taken |= 1u << (bc >> 5);
    float v = 0.f;
#pragma unroll
    for (int i = 0; i < kSmallTopkWarps; ++i)
      if (i == (bc >> 5)) v = cs[i];
    v = __shfl_sync(full, v, bc & 31);
    if (lane == j) {
      my_id = bi;
      my_sc = v;
    }
  }
  float total = lane < k ? my_sc : 0.f;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) total += __shfl_xor_sync(full, total, off);
  if (lane < k) {
    const float wgt = a.norm ? my_sc / total * a.scale : my_sc * a.scale;
    a.ids[(size_t)t * k + lane] = my_id;
    a.wts[(size_t)t * k + lane] = wgt;
    if (a.ids_out) a.ids_out[(size_t)t * k + lane] = my_id;
    if (a.wts_out) a.wts_out[(size_t)t * k + lane] = wgt;
    atomicAdd(&a.counts[my_id], 1);
    atomicOr(&a.bitmap[(size_t)my_id * a.W + (t >> 5)], 1u << (t & 31));
  }
}

// Few tokens (T <= kRouterGemvMaxT): the 64 x 64 tiles of router_logits_kernel
// would hold one or a few valid tokens and need a split-K sum, so instead one
// CTA per expert reads its router row once (float4 loads, 256 threads
// striding K) and accumulates every token's dot product; the 8 warps' sums
// are added in a fixed order (deterministic). One partial slice: splits = 1.
__global__ void __launch_bounds__(256) router_gemv_kernel(const __nv_bfloat16* __restrict__ x,
                                                          const float* __restrict__ W,
                                                          float* __restrict__ part, int T, int E,
                                                          int d) {
  __shared__ float red[8][kRouterGemvMaxT];
  const int e = blockIdx.x;
  const float* w = W + (size_t)e * d;
  float acc[kRouterGemvMaxT];
#pragma unroll
  for (int t = 0; t < kRouterGemvMaxT; ++t) acc[t] = 0.f;
  for (int c = threadIdx.x * 4; c < d; c += blockDim.x * 4) {
    const float4 wv = __ldg(reinterpret_cast<const float4*>(w + c));
#pragma unroll
    for (int t = 0; t < kRouterGemvMaxT; ++t) {
      if (t < T) {
        const uint2 raw = __ldg(reinterpret_cast<const uint2*>(x + (size_t)t * d + c));
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.x));
        const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.y));
        acc[t] = fmaf(a.x, wv.x, acc[t]);
        acc[t] = fmaf(a.y, wv.y, acc[t]);
        acc[t] = fmaf(b.x, wv.z, acc[t]);
        acc[t] = fmaf(b.y, wv.w, acc[t]);
      }
    }
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
  for (int t = 0; t < kRouterGemvMaxT; ++t) {
    float v = acc[t];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    if (lane == 0) red[warp][t] = v;
  }
  __syncthreads();
  if (threadIdx.x < T) {
    float sum = 0.f;
#pragma unroll
    for (int w8 = 0; w8 < 8; ++w8) sum += red[w8][threadIdx.x];
    part[(size_t)threadIdx.x * E + e] = sum;
  }
}

cudaError_t launch_router_logits(moe_handle* h, const void* x, int T, int splits, cudaStream_t s) {
  const Dims& dm = h->dims;
  if (T <= kRouterGemvMaxT) {  // the caller passes splits = 1 for these
    router_gemv_kernel<<<dm.E, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(x), h->w.router,
                                            h->ws.logits_part, T, dm.E, dm.d);
    h->launches++;
    return cudaGetLastError();
  }
  dim3 grid((dm.E + kRouterTile - 1) / kRouterTile, (T + kRouterTile - 1) / kRouterTile, splits);
  router_logits_kernel<<<grid, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(x), h->w.router,
                                            h->ws.logits_part, T, dm.E, dm.d,
                                            router_kps(dm, splits));
  h->launches++;
  return cudaGetLastError();
}

cudaError_t launch_router_topk(moe_handle* h, int T, int splits, const int32_t* forced,
                               cudaStream_t s, int32_t* ids_out, float* wts_out,
                               float* logits_out) {
  const Dims& dm = h->dims;
  const int W = static_cast<int>((dm.Tmax + 31) / 32);
  const int blocks = (T * 32 + 255) / 256;
  const TopkArgs a{h->ws.logits_part, splits, h->w.bias, T, dm.E, dm.k,
                   h->cfg.routed_scaling_factor, h->cfg.norm_topk_prob, forced, h->ws.ids,
                   h->ws.wts, h->ws.counts, h->ws.bitmap, W, h->ws.status, ids_out, wts_out,
                   logits_out, h->cfg.n_group, h->cfg.topk_group};
  if (T <= kSmallTopkMaxT && forced == nullptr && h->cfg.n_group == 1)
    router_topk_small_kernel<<<(T + 1) / 2, 256, 0, s>>>(a);
  else
    router_topk_kernel<<<blocks, 256, 0, s>>>(a);
  h->launches++;
  return cudaGetLastError();
}

// Both router kernels on caller-supplied buffers (no handle): used by the
// entry point that keeps its scratch in a static device array.
cudaError_t launch_router_raw(const void* x, const float* router_weight, const float* bias, int T,
                              int d, int E, int k, float scale, int norm, int splits, float* part,
                              int32_t* counts, uint32_t* bitmap, int W, uint32_t* status,
                              int32_t* ids, float* wts, cudaStream_t s) {
  Dims dm{};
  dm.d = d;
  dm.E = E;
  dim3 grid((E + kRouterTile - 1) / kRouterTile, (T + kRouterTile - 1) / kRouterTile, splits);
  router_logits_kernel<<<grid, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(x), router_weight,
                                            part, T, E, d, router_kps(dm, splits));
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int blocks = (T * 32 + 255) / 256;
  const TopkArgs a{part, splits, bias, T, E, k, scale, norm, nullptr, ids, wts, counts, bitmap,
                   W, status, nullptr, nullptr, nullptr, 1, 1};
  router_topk_kernel<<<blocks, 256, 0, s>>>(a);
  return cudaGetLastError();
}

// W_g (fp32 [E][d]) -> cat (BF16 [E][3d]) = [hi | mid | lo] with
// hi = bf16(w), mid = bf16(w - hi), lo = bf16(w - hi - mid); the differences
// are exact in fp32 and hi + mid + lo = w.
__global__ void router_split_kernel(const float* __restrict__ W, __nv_bfloat16* __restrict__ cat,
                                    int E, int d) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (int64_t)E * d) return;
  const int64_t e = i / d, c = i - e * d;
  const float w = W[i];
  const __nv_bfloat16 hi = __float2bfloat16_rn(w);
  const float r1 = w - __bfloat162float(hi);
  const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
  const float r2 = r1 - __bfloat162float(mid);
  const __nv_bfloat16 lo = __float2bfloat16_rn(r2);
  __nv_bfloat16* row = cat + e * 3 * (int64_t)d;
  row[c] = hi;
  row[d + c] = mid;
  row[2 * d + c] = lo;
}

cudaError_t launch_router_split(moe_handle* h, cudaStream_t s) {
  const Dims& dm = h->dims;
  const int64_t n = (int64_t)dm.E * dm.d;
  router_split_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, s>>>(
      h->w.router, static_cast<__nv_bfloat16*>(h->w.router_cat), dm.E, dm.d);
  h->launches++;
  return cudaGetLastError();
}

}  // namespace smoe
