// Token-to-expert dispatch and the weighted combine.
//
// The pages describe 384 independent experts that each see only their own
// tokens ("Kimi K2 · Down projection": 384 routed experts, each its own
// SwiGLU MLP); how tokens are grouped per expert is this library's design:
//
//   rows: every (token, slot) pair routed to expert e gets one row, and the
//   rows of expert e are contiguous [offsets[e], offsets[e+1]) in ascending
//   token order. The shared expert (split into n_shared groups of
//   moe_intermediate_size each) follows as groups E.., each holding all T
//   tokens in order.
//
// route_scan_kernel (one CTA): exclusive scan of the per-group row counts
//   into offsets; the GEMM work-unit prefix for both grouped GEMMs; and for
//   every expert the running popcount of its token bitmap words, so a pair's
//   rank inside its expert is one popcount away.
// dispatch: places every (token, slot) pair (pair_row, row_token). For row
//   tiles up to kGatherMaxBn rows the gate/up GEMMs gather each tile's token
//   rows straight from x with TMA (tile::gather4), so nothing is copied
//   (FP8: each token's x row is quantised once); taller tiles read the rows
//   copied here into expert order (FP8: quantised per row). Quantisation:
//   per 128 columns s = amax/448 and q = e4m3(x/s), both divisions
//   correctly rounded, conversion nearest-even and saturating.
// combine_kernel: y[t] = sum_j w[t,j] * out[row(t,j)] + sum_s out[shared
//   row(s,t)] over the BF16 per-row outputs, summed in fp32 in slot order and
//   rounded once to BF16.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "internal.h"
#include "route_common.cuh"

namespace smoe {

static int pick_bn(double want, const int* cands, int n, int cap = 1 << 30) {
  int last = cands[0];
  for (int i = 0; i < n && cands[i] <= cap; ++i) {
    last = cands[i];
    if (cands[i] >= want) return cands[i];
  }
  return last;
}

// Row-tile height: the smallest supported height >= SMOE_BN_FACTOR x the mean
// rows per routed expert, so that nearly every expert's rows fit one tile and
// each weight slab is read into shared memory once per forward. A taller cap
// costs no MMA work (each tile's N is its own row count rounded to 16 or 32),
// only pipeline depth and TMEM buffering; measured against 1.5: FP8 T=1024
// 3.97 -> 3.69 ms, BF16 T=1024 5.74 -> 5.36 ms, the bench's other sizes
// unchanged (their tiles are the same).
#ifndef SMOE_BN_FACTOR
#define SMOE_BN_FACTOR 3.0  // tuning constant
#endif
// FP8 gate/up tiles up to this height gather their token rows from the
// once-quantised x (taller FP8 tiles are bound by the promotion, not by TMA
// issue, so gathering may pay there too: a tuning constant)
#ifndef SMOE_FP8_GATHER_MAX_BN
#define SMOE_FP8_GATHER_MAX_BN 32
#endif
// tallest FP8 row tiles (tuning constants): gate/up 96 (three promotion
// warpgroups, two TMEM partial buffers), down 192. Measured against shorter
// caps at T = 16384 (same box): gate/up capped at 64 rows with four
// promotion warpgroups (four partial buffers) 12.30 vs 11.38 ms; down capped
// at 128 rows (four partial buffers) 7.50 vs 6.32 ms; T = 4096 likewise.
#ifndef SMOE_FP8_GU_MAX_BN
#define SMOE_FP8_GU_MAX_BN 96
#endif
#ifndef SMOE_FP8_DOWN_MAX_BN
#define SMOE_FP8_DOWN_MAX_BN 192
#endif
// mean rows per routed expert (T k / E); every token's row in each shared
// group when there are no routed experts
static double rows_per_group(const Dims& dm, int64_t T) {
  return dm.E > 0 ? static_cast<double>(T) * dm.k / dm.E : static_cast<double>(T);
}

GemmPlan plan_gate_up(const Dims& dm, int64_t T) {
  static const int bf16_bn[] = {16, 32, 64, 96, 128, 160, 192, 224, 256};
  static const int fp8_bn[] = {16, 32, 64, 96};
  const double want = SMOE_BN_FACTOR * rows_per_group(dm, T);
  GemmPlan p;
  p.bn = dm.fp8 ? pick_bn(want, fp8_bn, 4, SMOE_FP8_GU_MAX_BN) : pick_bn(want, bf16_bn, 9);
  p.na = 2;
  p.pair = !dm.fp8 && pair_bn_supported(p.bn) && dm.f % 256 == 0;
  p.gather = !p.pair && p.bn <= (dm.fp8 ? SMOE_FP8_GATHER_MAX_BN : kGatherMaxBn);
  p.m_tiles = dm.f / (p.pair ? 256 : kBlock);
  p.k_blocks = dm.fp8 ? dm.d / 128 : dm.d / 64;
  return p;
}

// Down projection: one unit covers 256 output features, as two 128-row
// weight tiles sharing the row tile (BF16 row tiles 64-96 on one SM; FP8 row
// tiles up to 64), so that every pipeline stage carries two weight tiles as
// the gate/up stage does, or (BF16 row tiles of 128 and more) as one pair MMA
// over a CTA pair.
GemmPlan plan_down(const Dims& dm, int64_t T) {
  static const int bf16_bn[] = {16, 32, 64, 96, 128, 160, 192, 224, 256};
  static const int fp8_bn[] = {16, 32, 64, 128, 192};
  const double want = SMOE_BN_FACTOR * rows_per_group(dm, T);
  GemmPlan p;
  p.bn = dm.fp8 ? pick_bn(want, fp8_bn, 5, SMOE_FP8_DOWN_MAX_BN) : pick_bn(want, bf16_bn, 9);
  p.pair = !dm.fp8 && pair_bn_supported(p.bn) && dm.d % 256 == 0 && dm.f % 128 == 0;
  p.gather = false;  // h rows are written in expert order by gate/up
  // two weight tiles per unit: FP8 up to 64 rows (measured: T=128 down GEMM
  // 1.05 -> 0.80 ms); BF16 from 64 rows (at 16 rows it changed nothing)
  p.na = (!p.pair && dm.d % 256 == 0 && (dm.fp8 ? p.bn <= 64 : p.bn >= 64)) ? 2 : 1;
  p.m_tiles = dm.d / (p.pair ? 256 : kBlock * p.na);
  p.k_blocks = dm.fp8 ? dm.f / 128 : dm.f / 64;
  return p;
}

// --------------------------------------------------------------- route scan
constexpr int kScanThreads = 1024;

__device__ __forceinline__ int block_exclusive_scan(int v, int* tmp, int* total) {
  // Hillis-Steele inclusive scan over the CTA, then shift to exclusive.
  const int tid = threadIdx.x;
  tmp[tid] = v;
  __syncthreads();
  for (int off = 1; off < kScanThreads; off <<= 1) {
    const int add = tid >= off ? tmp[tid - off] : 0;
    __syncthreads();
    tmp[tid] += add;
    __syncthreads();
  }
  const int incl = tmp[tid];
  *total = tmp[kScanThreads - 1];
  __syncthreads();
  return incl - v;
}

// CTA 0 scans the per-group counts; CTAs 1.. compute, one warp per expert,
// the running popcount of the expert's token bitmap over the words that can
// hold tokens (ceil(T / 32) of the row's W).
__global__ void __launch_bounds__(kScanThreads) route_scan_kernel(
    const int32_t* __restrict__ counts, int E, int ns, int T, const uint32_t* __restrict__ bitmap,
    int W, int32_t* __restrict__ word_prefix, int32_t* __restrict__ offsets,
    int32_t* __restrict__ unit_base, int bn1, int mt1, int bn2, int mt2) {
  if (blockIdx.x == 0) {
    __shared__ int tmp[kScanThreads];
    const int G = E + ns;
    const int g = threadIdx.x;  // G <= kMaxExperts + 16 < 1024
    int c = 0;
    if (g < E) c = counts[g];
    else if (g < G) c = T;
    const int u1 = mt1 * ((c + bn1 - 1) / bn1);
    const int u2 = mt2 * ((c + bn2 - 1) / bn2);
    int tot;
    const int o = block_exclusive_scan(c, tmp, &tot);
    if (g <= G) offsets[g] = o;
    const int b1 = block_exclusive_scan(u1, tmp, &tot);
    if (g <= G) unit_base[g] = b1;
    const int b2 = block_exclusive_scan(u2, tmp, &tot);
    if (g <= G) unit_base[(G + 1) + g] = b2;
    return;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int e = (blockIdx.x - 1) * (kScanThreads / 32) + warp;
  if (e >= E) return;
  const int words = (T + 31) / 32;
  int run = 0;
  for (int w0 = 0; w0 < words; w0 += 32) {
    const int w = w0 + lane;
    const int v = w < words ? __popc(bitmap[(size_t)e * W + w]) : 0;
    int incl = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += n;
    }
    if (w < words) word_prefix[(size_t)e * W + w] = run + incl - v;
    run += __shfl_sync(0xffffffffu, incl, 31);
  }
}

cudaError_t launch_route_scan(moe_handle* h, int T, const GemmPlan& p1, const GemmPlan& p2,
                              cudaStream_t s) {
  const Dims& dm = h->dims;
  const int W = static_cast<int>((dm.Tmax + 31) / 32);
  const int blocks = 1 + (dm.E + kScanThreads / 32 - 1) / (kScanThreads / 32);
  route_scan_kernel<<<blocks, kScanThreads, 0, s>>>(
      h->ws.counts, dm.E, dm.ns, T, h->ws.bitmap, W, h->ws.word_prefix, h->ws.offsets,
      h->ws.unit_base, p1.bn, p1.m_tiles, p2.bn, p2.m_tiles);
  h->launches++;
  return cudaGetLastError();
}

// ----------------------------------------------------------------- dispatch
// Tall row tiles: one warp per row places the pair (pair_row, row_token)
// and copies the token's x row into the gathered matrix in row order with
// 16-byte loads and stores (FP8: quantises it on the way, as below).
__global__ void __launch_bounds__(256) dispatch_bf16_kernel(
    const __nv_bfloat16* __restrict__ x, int T, int d, int k, int E, int items,
    const int32_t* __restrict__ ids, const uint32_t* __restrict__ bitmap,
    const int32_t* __restrict__ word_prefix, const int32_t* __restrict__ offsets, int W,
    int32_t* __restrict__ pair_row, int32_t* __restrict__ row_token,
    __nv_bfloat16* __restrict__ xp) {
  const int lane = threadIdx.x & 31;
  const int i = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (i >= items) return;
  int t;
  const int row = place_row(i, T, k, E, ids, bitmap, word_prefix, offsets, W, &t);
  if (lane == 0) {
    if (i < T * k) pair_row[i] = row;
    row_token[row] = t;
  }
  const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t * d);
  uint4* dst = reinterpret_cast<uint4*>(xp + (size_t)row * d);
  const int n16 = d / 8;  // a multiple of 16 (d is a multiple of 128)
  // four 16-byte loads in flight per lane before their stores
  for (int c = lane; c < n16; c += 128) {
    uint4 v[4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if (c + 32 * j < n16) v[j] = __ldg(src + c + 32 * j);
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if (c + 32 * j < n16) dst[c + 32 * j] = v[j];
  }
}

__global__ void __launch_bounds__(256) dispatch_fp8_kernel(
    const __nv_bfloat16* __restrict__ x, int T, int d, int k, int E, int items,
    const int32_t* __restrict__ ids, const uint32_t* __restrict__ bitmap,
    const int32_t* __restrict__ word_prefix, const int32_t* __restrict__ offsets, int W,
    int32_t* __restrict__ pair_row, int32_t* __restrict__ row_token, uint8_t* __restrict__ xq,
    float* __restrict__ xs) {
  const int lane = threadIdx.x & 31;
  const int i = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (i >= items) return;
  int t;
  const int row = place_row(i, T, k, E, ids, bitmap, word_prefix, offsets, W, &t);
  if (lane == 0) {
    if (i < T * k) pair_row[i] = row;
    row_token[row] = t;
  }
  quant_row_e4m3(x + (size_t)t * d, d, xq + (size_t)row * d, xs + (size_t)row * (d / 128), lane);
}

// Short row tiles: one thread per (token, slot) pair and per shared-group
// row (blocks [0, place_blocks)) writes the pair's row (pair_row) and the
// row's token (row_token), which the gate/up GEMMs use to gather x rows; no
// row is copied. FP8: the blocks after those quantise each token's x row
// once (qparts warps per token) into rows [0, T) of xq / xs, which the GEMMs
// gather from instead of x.
__global__ void __launch_bounds__(256) dispatch_kernel(
    const __nv_bfloat16* __restrict__ x, int T, int d, int k, int E, int items, int place_blocks,
    int qparts,
    const int32_t* __restrict__ ids, const uint32_t* __restrict__ bitmap,
    const int32_t* __restrict__ word_prefix, const int32_t* __restrict__ offsets, int W,
    int32_t* __restrict__ pair_row, int32_t* __restrict__ row_token, uint8_t* __restrict__ xq,
    float* __restrict__ xs) {
  if (static_cast<int>(blockIdx.x) < place_blocks) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= items) return;
    int t;
    const int row = place_row(i, T, k, E, ids, bitmap, word_prefix, offsets, W, &t);
    if (i < T * k) pair_row[i] = row;
    row_token[row] = t;
    return;
  }
  const int lane = threadIdx.x & 31;
  const int qw = ((blockIdx.x - place_blocks) * blockDim.x + threadIdx.x) >> 5;
  const int t = qw / qparts;
  if (t >= T) return;
  quant_row_e4m3(x + (size_t)t * d, d, xq + (size_t)t * d, xs + (size_t)t * (d / 128), lane,
                 qw - t * qparts, qparts);
}

// Dynamic activation quantisation of a dense [rows, d] BF16 matrix.
__global__ void __launch_bounds__(256) act_quant_kernel(const __nv_bfloat16* __restrict__ x,
                                                        int64_t rows, int d, int parts,
                                                        uint8_t* __restrict__ q,
                                                        float* __restrict__ s) {
  const int lane = threadIdx.x & 31;
  const int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t r = w / parts;
  if (r >= rows) return;
  quant_row_e4m3(x + r * d, d, q + r * d, s + r * (d / 128), lane, static_cast<int>(w - r * parts),
                 parts);
}

// Warps per row of the e4m3 quantisation: one per row when there are rows
// enough to fill the GPU (~16 warps per SM), else up to one per pair of
// 128-column groups.
static int quant_parts(int64_t rows, int d, int sms = 148) {
  const int64_t want = 16 * static_cast<int64_t>(sms);
  const int64_t most = (d / 128 + 1) / 2;
  const int64_t p = rows > 0 ? want / rows : most;
  return static_cast<int>(p < 1 ? 1 : (p > most ? most : p));
}

cudaError_t launch_act_quant(const void* x, int64_t rows, int d, uint8_t* q, float* s,
                             cudaStream_t st) {
  const int parts = quant_parts(rows, d);
  const int64_t blocks = (rows * parts * 32 + 255) / 256;
  act_quant_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(x), rows, d, parts, q, s);
  return cudaGetLastError();
}

cudaError_t launch_dispatch(moe_handle* h, const void* x, int T, bool gather, cudaStream_t s) {
  const Dims& dm = h->dims;
  const int W = static_cast<int>((dm.Tmax + 31) / 32);
  const int items = T * (dm.k + dm.ns);
  const __nv_bfloat16* xb = static_cast<const __nv_bfloat16*>(x);
  if (gather) {
    const int place_blocks = (items + 255) / 256;
    const int qparts = dm.fp8 ? quant_parts(T, dm.d, h->num_sms) : 1;
    const int quant_blocks =
        dm.fp8 ? static_cast<int>(((int64_t)T * qparts * 32 + 255) / 256) : 0;
    dispatch_kernel<<<place_blocks + quant_blocks, 256, 0, s>>>(
        xb, T, dm.d, dm.k, dm.E, items, place_blocks, qparts, h->ws.ids, h->ws.bitmap,
        h->ws.word_prefix, h->ws.offsets, W, h->ws.pair_row, h->ws.row_token,
        static_cast<uint8_t*>(h->ws.xp), h->ws.xs);
  } else {
    const int blocks = static_cast<int>(((int64_t)items * 32 + 255) / 256);
    if (dm.fp8) {
      dispatch_fp8_kernel<<<blocks, 256, 0, s>>>(
          xb, T, dm.d, dm.k, dm.E, items, h->ws.ids, h->ws.bitmap, h->ws.word_prefix,
          h->ws.offsets, W, h->ws.pair_row, h->ws.row_token, static_cast<uint8_t*>(h->ws.xp),
          h->ws.xs);
    } else {
      dispatch_bf16_kernel<<<blocks, 256, 0, s>>>(
          xb, T, dm.d, dm.k, dm.E, items, h->ws.ids, h->ws.bitmap, h->ws.word_prefix,
          h->ws.offsets, W, h->ws.pair_row, h->ws.row_token,
          static_cast<__nv_bfloat16*>(h->ws.xp));
    }
  }
  h->launches++;
  return cudaGetLastError();
}

// ------------------------------------------------------------------ combine
// 8 columns per thread: one 16-byte load per expert row, one 16-byte store.
constexpr int kCombineThreads = 128;

constexpr int kSmallCombineMaxT = 256;

// U > 1 (few tokens): the slots are taken U at a time, their row indices and
// then their rows loaded together, one load latency per batch instead of two
// per slot (the sum keeps slot order). Many tokens keep U = 1: there the
// kernel streams HBM and the batched form measured slower (0.215 -> 0.272 ms
// at T = 8192; decode T = 64 11.5 -> 9.7 us).
template <int U>
__global__ void __launch_bounds__(kCombineThreads)
    combine_kernel(const uint16_t* __restrict__ out, const int32_t* __restrict__ pair_row,
                   const float* __restrict__ wts, const int32_t* __restrict__ offsets, int T, int d,
                   int k, int E, int ns, __nv_bfloat16* __restrict__ y) {
  const int t = blockIdx.x;
  const int c = (blockIdx.y * blockDim.x + threadIdx.x) * 8;
  if (c >= d) return;
  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;
  if (U == 1) {
    for (int j = 0; j < k; ++j) {
      const int row = pair_row[(size_t)t * k + j];
      add_row8(acc, out + (size_t)row * d + c, wts[(size_t)t * k + j]);
    }
  } else {
    for (int j0 = 0; j0 < k; j0 += U) {
      int row[U];
      float w[U];
      uint4 v[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        if (j0 + u < k) {
          row[u] = __ldg(pair_row + (size_t)t * k + j0 + u);
          w[u] = __ldg(wts + (size_t)t * k + j0 + u);
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u)
        if (j0 + u < k) v[u] = __ldg(reinterpret_cast<const uint4*>(out + (size_t)row[u] * d + c));
#pragma unroll
      for (int u = 0; u < U; ++u)
        if (j0 + u < k) add_row8v(acc, v[u], w[u]);
    }
  }
  for (int s = 0; s < ns; ++s) add_row8(acc, out + (size_t)(offsets[E + s] + t) * d + c, 1.f);
  uint32_t pk[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    __nv_bfloat162 b = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
    pk[i] = *reinterpret_cast<uint32_t*>(&b);
  }
  *reinterpret_cast<uint4*>(y + (size_t)t * d + c) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
}

cudaError_t launch_combine(moe_handle* h, void* y, int T, cudaStream_t s) {
  const Dims& dm = h->dims;
  dim3 grid(T, (dm.d / 8 + kCombineThreads - 1) / kCombineThreads);
  auto kern = T <= kSmallCombineMaxT ? combine_kernel<8> : combine_kernel<1>;
  kern<<<grid, kCombineThreads, 0, s>>>(h->ws.out, h->ws.pair_row, h->ws.wts, h->ws.offsets, T,
                                        dm.d, dm.k, dm.E, dm.ns, static_cast<__nv_bfloat16*>(y));
  h->launches++;
  return cudaGetLastError();
}

// ------------------------------------------------------- combine of rows
// The combine step on rows already in (token, slot) order: the last step of
// an expert-parallel forward, after each pair's output came back from the
// rank that owns its expert. Same arithmetic as combine_kernel.
__global__ void __launch_bounds__(kCombineThreads)
    combine_rows_kernel(const uint16_t* __restrict__ pair_out, const float* __restrict__ wts,
                        const uint16_t* __restrict__ shared, int T, int d, int k,
                        __nv_bfloat16* __restrict__ y) {
  const int t = blockIdx.x;
  const int c = (blockIdx.y * blockDim.x + threadIdx.x) * 8;
  if (c >= d) return;
  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;
  for (int j = 0; j < k; ++j)
    add_row8(acc, pair_out + ((size_t)t * k + j) * d + c, wts[(size_t)t * k + j]);
  if (shared) add_row8(acc, shared + (size_t)t * d + c, 1.f);
  uint32_t pk[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    __nv_bfloat162 b = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
    pk[i] = *reinterpret_cast<uint32_t*>(&b);
  }
  *reinterpret_cast<uint4*>(y + (size_t)t * d + c) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
}

cudaError_t launch_combine_rows(const void* pair_out, const float* wts, const void* shared, int T,
                                int d, int k, void* y, cudaStream_t s) {
  dim3 grid(T, (d / 8 + kCombineThreads - 1) / kCombineThreads);
  combine_rows_kernel<<<grid, kCombineThreads, 0, s>>>(
      static_cast<const uint16_t*>(pair_out), wts, static_cast<const uint16_t*>(shared), T, d, k,
      static_cast<__nv_bfloat16*>(y));
  return cudaGetLastError();
}

}  // namespace smoe
