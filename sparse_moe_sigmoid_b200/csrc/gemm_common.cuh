// Pieces shared by the BF16 and FP8 grouped GEMM kernels: the work-unit
// decoding and the shared-memory carve-up.
//
// Work decomposition (both GEMMs of the expert MLP): the output of group g
// (an expert, or a slice of the shared expert) is a [features x rows]
// matrix, rows = the tokens routed to g. It is cut into tiles of 128
// features x BN rows. A unit is one such tile; units are numbered group by
// group, feature tile by feature tile, row tile innermost, so units that use
// the same 128-row weight slab are adjacent and run at the same time on
// neighbouring CTAs, which then read the slab from HBM once and from L2
// after that. CTA c takes units c, c + gridDim.x, ... (persistent grid).
#pragma once

#include <stdint.h>

#include "sm100.cuh"

namespace smoe {

struct Unit {
  int g;       // group (expert)
  int mt;      // 128-feature tile
  int row0;    // first row of the row tile
  int nvalid;  // rows of the tile that belong to g (1..BN)
  int split;   // K slice (single-group mode with ksplit > 1), else 0
};

struct GemmArgs {
  const int32_t* offsets;    // [G+1]
  const int32_t* unit_base;  // [G+1] prefix of units per group
  int G;
  int m_tiles;
  int k_blocks;
  int bn;
  void* out;                 // gate/up: h [R][ld]; down: BF16 out [R][ld]; router: fp32
  int ld;
  float* out_scale;          // FP8 gate/up: h scales [R][f/128]
  const float* w_scale0;     // FP8: weight block scales of A0 [G][m_tiles][k_blocks]
  const float* w_scale1;     // FP8 gate/up: of A1
  const float* act_scale;    // FP8: activation scales [R][k_blocks]
  uint32_t* status;
  int single_rows;           // unit_base == nullptr: one group of this many rows at row 0
  int b_k;                   // K extent of B; the K index into B is (k mod b_k)
  int m_valid;               // only output features < m_valid are stored
  int kpp;                   // promoted BF16 GEMM: stages accumulated in TMEM per promotion
  int kpp_rest;              // the same for K slices after the first (0: kpp)
  int stages;                // promoted GEMM: shared-memory ring depth
  int32_t* sched;            // pair GEMM: unit counter, zero at launch (dynamic units); null: static
  int ksplit;                // single-group mode: K slices per tile (0 or 1: none); slice s
                             // covers k-blocks [s, s+1) * k_blocks / ksplit and writes its
                             // partial result at out + s * split_stride elements
  size_t split_stride;
  int out_bf16;               // promoted GEMM, plain mode: outputs stored BF16 (else fp32)
  uint64_t wait_ns;           // limit of each pipeline wait (the wind-down keeps the default)
  int stall;                  // test hook: the MMA issuer waits on a barrier nothing signals
  // gathered B (gate/up): row i of a tile is row row_token[row0 + i] of the B
  // tensor (the token's x row), loaded four rows per tile::gather4; null: the
  // B rows are the tile's own rows [row0, row0 + BN) of B (down, router)
  const int32_t* row_token;
};

// Token rows of B for rows [r, r + 4) of a gathered tile whose valid rows end
// at `end` (rows past it repeat the tile's first row: they are loaded so that
// the MMA's N stays a multiple of 16, and their outputs are never stored).
__device__ __forceinline__ void gather_rows(const GemmArgs& a, int row0, int r, int end,
                                            int (&tok)[4]) {
#pragma unroll
  for (int j = 0; j < 4; ++j) tok[j] = __ldg(a.row_token + (r + j < end ? r + j : row0));
}

// Limit of a pipeline wait: the caller's, or the default.
__device__ __forceinline__ uint64_t wait_limit(const GemmArgs& a) {
  return a.wait_ns ? a.wait_ns : sm100::kTimeoutNs;
}

__device__ __forceinline__ int total_units_of(const GemmArgs& a, int BN) {
  return a.unit_base ? __ldg(a.unit_base + a.G)
                     : a.m_tiles * ((a.single_rows + BN - 1) / BN) * (a.ksplit > 1 ? a.ksplit : 1);
}

__device__ __forceinline__ Unit decode_unit(int u, const GemmArgs& a, int BN) {
  Unit un;
  un.split = 0;
  if (a.unit_base == nullptr) {
    if (a.ksplit > 1) {  // the K slices of one tile are adjacent units
      un.split = u % a.ksplit;
      u /= a.ksplit;
    }
    const int nt = (a.single_rows + BN - 1) / BN;
    un.g = 0;
    un.mt = u / nt;
    const int ti = u - un.mt * nt;
    un.row0 = ti * BN;
    un.nvalid = min(BN, a.single_rows - ti * BN);
    return un;
  }
  // last group whose first unit is <= u (empty groups own no units)
  int lo = 0, hi = a.G;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (__ldg(a.unit_base + mid) <= u) lo = mid;
    else hi = mid;
  }
  un.g = lo;
  const int r0 = __ldg(a.offsets + lo);
  const int cnt = __ldg(a.offsets + lo + 1) - r0;
  const int nt = (cnt + BN - 1) / BN;
  const int local = u - __ldg(a.unit_base + lo);
  un.mt = local / nt;
  const int ti = local - un.mt * nt;
  un.row0 = r0 + ti * BN;
  un.nvalid = min(BN, cnt - ti * BN);
  return un;
}

__host__ __device__ constexpr int pow2_at_least(int v, int lo) {
  int p = lo;
  while (p < v) p <<= 1;
  return p;
}

}  // namespace smoe
