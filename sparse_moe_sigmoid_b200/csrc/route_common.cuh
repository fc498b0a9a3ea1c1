// Per-token arithmetic shared by the phase kernels (router.cu, dispatch.cu)
// and the single-launch small-batch layer (layer_small.cu): the noaux_tc
// top-k of one token (with the group filter), the placement of a (token,
// slot) pair in the grouped GEMMs' row order, the dynamic e4m3 quantisation
// of one row, and one 8-column step of the weighted combine.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <math.h>

#include "internal.h"

namespace smoe {

constexpr int kPerLane = kMaxExperts / 32;

// Group-limited routing (n_group > 1; "Kimi K2 Base" raw config fields
// n_group / topk_group, both 1 for K2, whose config post, §2.4, explains what
// grouping is for). The experts form n_group contiguous groups of E / n_group;
// a group scores the fp32 sum of its two largest keys (its one key for groups
// of one); the topk_group best groups are kept, ties to the lower group; the
// other groups' keys become -inf so that the top-k below never picks them.
// One warp: the keys go through this warp's shared-memory row, lane g < n_group
// scans group g, and the groups are picked by topk_group shuffle arg-max rounds.
__device__ __forceinline__ void group_filter(float (&key)[kMaxExperts / 32], int E, int n_group,
                                             int topk_group, float* __restrict__ row,
                                             int lane) {
  const unsigned full = 0xffffffffu;
#pragma unroll
  for (int i = 0; i < kMaxExperts / 32; ++i)
    if (lane + 32 * i < E) row[lane + 32 * i] = key[i];
  __syncwarp();
  const int gs = E / n_group;
  float gscore = -INFINITY;
  if (lane < n_group) {
    float b1 = -INFINITY, b2 = -INFINITY;  // the two largest keys of group `lane`
    for (int j = 0; j < gs; ++j) {
      const float v = row[lane * gs + j];
      if (v > b1) {
        b2 = b1;
        b1 = v;
      } else if (v > b2) {
        b2 = v;
      }
    }
    gscore = gs >= 2 ? b1 + b2 : b1;
  }
  uint32_t kept = 0;  // bit g: group g kept
  for (int r = 0; r < topk_group; ++r) {
    float bv = (lane < n_group && !((kept >> lane) & 1u)) ? gscore : -INFINITY;
    int bi = (lane < n_group && !((kept >> lane) & 1u)) ? lane : 0x7fffffff;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float ov = __shfl_xor_sync(full, bv, off);
      const int oi = __shfl_xor_sync(full, bi, off);
      if (ov > bv || (ov == bv && oi < bi)) {
        bv = ov;
        bi = oi;
      }
    }
    if (bi >= n_group) {  // NaN or -inf scores only: the lowest group not yet kept
      bi = 0;
      while (bi < n_group && ((kept >> bi) & 1u)) ++bi;
    }
    kept |= 1u << bi;
  }
#pragma unroll
  for (int i = 0; i < kMaxExperts / 32; ++i) {
    const int e = lane + 32 * i;
    if (e < E && !((kept >> (e / gs)) & 1u)) key[i] = -INFINITY;
  }
  __syncwarp();
}

// Arguments of the per-token top-k.
struct TopkArgs {
  const float* part;  // [splits][T][E] partial logits, added in slice order
  int splits;
  const float* bias;
  int T, E, k;
  float scale;
  int norm;
  const int32_t* forced;  // [T][k] forced ids, or null
  int32_t* ids;           // [T][k]
  float* wts;             // [T][k]
  int32_t* counts;        // [E]
  uint32_t* bitmap;       // [E][W]
  int W;
  uint32_t* status;
  int32_t* ids_out;
  float* wts_out;
  float* logits_out;
  int n_group, topk_group;
};

// Router of token t by one warp ("Kimi K2 Base" raw config: scoring_func
// sigmoid, topk_method noaux_tc, num_experts_per_tok, norm_topk_prob,
// routed_scaling_factor). Lane l holds experts l, l + 32, ...: it adds the
// partial logits, takes the sigmoid, forms the key score + bias, applies the
// group filter when n_group > 1, and the warp extracts the k largest keys
// (ties to the lower expert index) by k rounds of a shuffle arg-max. The
// weights use the unbiased scores: w = score / sum(selected scores) * scale.
// It also counts tokens per expert and sets the token's bit in the expert's
// bitmap. group_row: this warp's kMaxExperts floats of shared memory.
__device__ __forceinline__ void route_token(const TopkArgs& a, int t, float* group_row,
                                            int lane) {
  const float* __restrict__ part = a.part;
  const int splits = a.splits, T = a.T, E = a.E, k = a.k;
  const float* __restrict__ bias = a.bias;
  const int32_t* __restrict__ forced = a.forced;
  uint32_t* status = a.status;
  float* logits_out = a.logits_out;
  const unsigned full = 0xffffffffu;

  float key[kPerLane], sc[kPerLane], lg[kPerLane];
#pragma unroll
  for (int i = 0; i < kPerLane; ++i) lg[i] = 0.f;
  // slices in order (a deterministic sum); the loads of a slice's experts are
  // independent, so they are issued together, four slices at a time (plain
  // loads: the single-launch layer writes the logits in the same launch)
#pragma unroll 4
  for (int s = 0; s < splits; ++s) {
    const float* ps = part + ((size_t)s * T + t) * E;
    float v[kPerLane];
#pragma unroll
    for (int i = 0; i < kPerLane; ++i) v[i] = lane + 32 * i < E ? ps[lane + 32 * i] : 0.f;
#pragma unroll
    for (int i = 0; i < kPerLane; ++i) lg[i] += v[i];
  }
#pragma unroll
  for (int i = 0; i < kPerLane; ++i) {
    const int e = lane + 32 * i;
    if (e < E) {
      const float l = lg[i];
      if (logits_out) logits_out[(size_t)t * E + e] = l;
      const float p = 1.f / (1.f + expf(-l));
      sc[i] = p;
      key[i] = p + bias[e];
    } else {
      sc[i] = 0.f;
      key[i] = -INFINITY;
    }
  }

  int my_id = 0;
  float my_sc = 0.f;
  bool use_forced = forced != nullptr;
  if (use_forced) {
    int e = -1;
    if (lane < k) e = forced[(size_t)t * k + lane];
    bool bad = lane < k && (e < 0 || e >= E);
    for (int jj = 0; jj < k; ++jj) {
      const int other = __shfl_sync(full, e, jj);
      if (lane < k && jj < lane && other == e) bad = true;
    }
    if (__any_sync(full, bad)) {
      // an out-of-range or repeated id: report it and select normally, which
      // keeps the dispatch's bookkeeping consistent
      if (lane == 0) atomicOr(status, MOE_DEVICE_BAD_EXPERT_ID);
      use_forced = false;
    } else {
      // each lane j < k fetches its expert's score from the owning lane
      for (int jj = 0; jj < k; ++jj) {
        const int ej = __shfl_sync(full, e, jj);
        float v = 0.f;
#pragma unroll
        for (int i = 0; i < kPerLane; ++i)
          if (i == (ej >> 5)) v = sc[i];
        v = __shfl_sync(full, v, ej & 31);
        if (lane == jj) {
          my_id = ej;
          my_sc = v;
        }
      }
    }
  }
  if (!use_forced) {
    if (a.n_group > 1) group_filter(key, E, a.n_group, a.topk_group, group_row, lane);
    uint32_t taken = 0;  // bit i: expert lane + 32 i already chosen
    for (int j = 0; j < k; ++j) {
      float bk = -INFINITY;
      int bi = 0x7fffffff;
#pragma unroll
      for (int i = 0; i < kPerLane; ++i) {
        const int e = lane + 32 * i;
        if (e < E && !((taken >> i) & 1u) && (key[i] > bk || (key[i] == bk && e < bi))) {
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
      if (bi >= E) {  // NaN keys: nothing comparable left; keep the bookkeeping valid
        if (lane == 0) atomicOr(status, MOE_DEVICE_BAD_EXPERT_ID);
        bi = 0;
        while (bi < E) {  // smallest id not yet taken
          const int owner = bi & 31;
          const uint32_t tk = __shfl_sync(full, taken, owner);
          if (!((tk >> (bi >> 5)) & 1u)) break;
          ++bi;
        }
      }
      if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
      float v = 0.f;
#pragma unroll
      for (int i = 0; i < kPerLane; ++i)
        if (i == (bi >> 5)) v = sc[i];
      v = __shfl_sync(full, v, bi & 31);
      if (lane == j) {
        my_id = bi;
        my_sc = v;
      }
    }
  }

  float total = lane < k ? my_sc : 0.f;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) total += __shfl_xor_sync(full, total, off);
  if (lane < k) {
    const float w = a.norm ? my_sc / total * a.scale : my_sc * a.scale;
    a.ids[(size_t)t * k + lane] = my_id;
    a.wts[(size_t)t * k + lane] = w;
    if (a.ids_out) a.ids_out[(size_t)t * k + lane] = my_id;
    if (a.wts_out) a.wts_out[(size_t)t * k + lane] = w;
    atomicAdd(&a.counts[my_id], 1);
    atomicOr(&a.bitmap[(size_t)my_id * a.W + (t >> 5)], 1u << (t & 31));
  }
}

__device__ __forceinline__ int place_row(int i, int T, int k, int E, const int32_t* ids,
                                         const uint32_t* bitmap, const int32_t* word_prefix,
                                         const int32_t* offsets, int W, int* tok) {
  const int nrouted = T * k;
  if (i < nrouted) {
    const int t = i / k;
    const int e = ids[i];
    const int w = t >> 5;
    const uint32_t below = bitmap[(size_t)e * W + w] & ((1u << (t & 31)) - 1u);
    *tok = t;
    return offsets[e] + word_prefix[(size_t)e * W + w] + __popc(below);
  }
  const int s = (i - nrouted) / T;
  const int t = (i - nrouted) % T;
  *tok = t;
  return offsets[E + s] + t;
}

// One row of d BF16 values -> d e4m3 codes + d/128 fp32 scales: each
// half-warp takes one 128-column group (16 lanes x 8 values). A row may be
// shared by `parts` warps, warp `part` taking the group pairs part,
// part + parts, ... (few rows: the groups' loads then run in parallel
// instead of one after another in a single warp).
__device__ __forceinline__ void quant_row_e4m3(const __nv_bfloat16* __restrict__ src, int d,
                                               uint8_t* __restrict__ dst,
                                               float* __restrict__ scales, int lane,
                                               int part = 0, int parts = 1) {
  const int ngroups = d / 128;
  for (int g0 = 2 * part; g0 < ngroups; g0 += 2 * parts) {
    const int gi = g0 + (lane >> 4);
    const bool active = gi < ngroups;
    const int col = gi * 128 + (lane & 15) * 8;
    float v[8];
    float amax = 0.f;
    if (active) {
      const uint4 raw = __ldg(reinterpret_cast<const uint4*>(src + col));
      const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 f2 = __bfloat1622float2(p[j]);
        v[2 * j] = f2.x;
        v[2 * j + 1] = f2.y;
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fabsf(v[j]));
    }
#pragma unroll
    for (int off = 8; off > 0; off >>= 1)
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    if (active) {
      const float sa = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
      uint32_t packed[2];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float2 q;
        q.x = __fdiv_rn(v[2 * j], sa);
        q.y = __fdiv_rn(v[2 * j + 1], sa);
        const __nv_fp8x2_storage_t b = __nv_cvt_float2_to_fp8x2(q, __NV_SATFINITE, __NV_E4M3);
        if (j & 1) packed[j >> 1] |= static_cast<uint32_t>(b) << 16;
        else packed[j >> 1] = static_cast<uint32_t>(b);
      }
      *reinterpret_cast<uint2*>(dst + col) = make_uint2(packed[0], packed[1]);
      if ((lane & 15) == 0) scales[gi] = sa;
    }
  }
}

// acc += w * (8 BF16 values packed in v)
__device__ __forceinline__ void add_row8v(float (&acc)[8], const uint4 v, float w) {
  const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {  // BF16 -> fp32 is exact: the bits move up by 16
    acc[2 * i] = fmaf(w, __uint_as_float(u[i] << 16), acc[2 * i]);
    acc[2 * i + 1] = fmaf(w, __uint_as_float(u[i] & 0xFFFF0000u), acc[2 * i + 1]);
  }
}

// NC: read through the read-only path (the rows were written by an earlier
// launch); the single-launch layer reads rows of its own launch coherently.
template <bool NC = true>
__device__ __forceinline__ void add_row8(float (&acc)[8], const uint16_t* p, float w) {
  const uint4 v = NC ? __ldg(reinterpret_cast<const uint4*>(p)) : *reinterpret_cast<const uint4*>(p);
  add_row8v(acc, v, w);
}

}  // namespace smoe
