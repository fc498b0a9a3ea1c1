// Grouped expert GEMMs, BF16 weights, on the sm_100a tensor cores.
//
// Expert MLP ("Kimi K2 · Down projection", OpenModelAtlas: the module
// formula down_proj(act_fn(gate_proj(x)) * up_proj(x)), weights [out, in],
// no bias; act_fn = silu from the config's hidden_act):
//   gate/up: h[r, :] = silu(W_gate x_r) * (W_up x_r)   W_gate, W_up [f, d]
//   down:    out[r, :] = W_down h_r                     W_down [d, f]
// for every row r of a group (the rows routed to one expert).
//
// Both run as D = A . B^T with A = a 128-row slab of the weight (K-major,
// straight from the [out, in] layout) and B = BN gathered activation rows
// (K-major). The weight is the operand that fills the 128-wide M side, so a
// group with few tokens (decode: about 2 per expert) still uses full-size
// MMAs, and N = the group's row count rounded up to 16 is set per tile in
// the instruction descriptor; nothing is padded to a token tile of 128.
//
// One persistent CTA per SM, 6 warps:
//   warp 0      TMA producer: A (gate, and up for the gated GEMM) and B tiles
//               of 64 K-columns into a ring of smem stages (128-byte swizzle).
//   warp 1      allocates TMEM and issues tcgen05.mma (K = 16 per
//               instruction, 4 per stage) into a double-buffered fp32
//               accumulator; tcgen05.commit releases stages and hands
//               finished accumulators to the epilogue.
//   warps 2..5  epilogue: tcgen05.ld of the accumulator (TMEM lane = output
//               feature, column = row), then SwiGLU and a BF16 store of h, or
//               a BF16 store of the down projection's per-row output. The
//               second accumulator buffer lets the next tile's MMAs run
//               meanwhile.
// Every wait is bounded (2 s); a wait that runs out sets
// MOE_DEVICE_WAIT_TIMEOUT in the status word and the CTA winds down: it
// waits (bounded) for its own loads and MMAs in flight, frees TMEM and
// returns.
#include <cuda_bf16.h>

#include "gemm_common.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace smoe {

using namespace sm100;

// NA = weight tiles per stage (2: gate and up for SWIGLU, or two 128-row
// halves of one 256-feature tile for the plain store). The accumulators are
// double-buffered in TMEM when two sets fit in its 512 columns, else single.
template <int BN, int NA, bool SWIGLU>
struct Bf16Cfg {
  static constexpr int kA = 128 * 64 * 2;  // one 128 x 64 BF16 weight tile
  static constexpr int kB = BN * 64 * 2;
  static constexpr int kNumA = NA;
  static constexpr int kStage = kA * kNumA + kB;
  static constexpr int kStages0 = (227 * 1024 - 2048) / kStage;
  static constexpr int kStages = kStages0 > 12 ? 12 : kStages0;
  static constexpr int kAccCols = NA * BN;
  static constexpr int kAccBufs = 2 * kAccCols <= 512 ? 2 : 1;
  static constexpr int kTmemCols = pow2_at_least(kAccBufs * kAccCols, 32);
  static constexpr int kSmem = kStages * kStage + 1024 + 256;  // + barriers and flags
  static_assert(kStage % 1024 == 0, "stage must keep 1024-byte alignment");
  static_assert(kTmemCols <= 512, "TMEM holds 512 columns");
  static_assert(kStages >= 2, "need at least two stages");
  static_assert(!SWIGLU || NA == 2, "SwiGLU needs the gate and up tiles");
  static_assert(BN <= 256, "a gathered tile takes at most two gather4 per lane");
};

template <int BN, int NA, bool SWIGLU>
__global__ void __launch_bounds__(192, 1)
    grouped_gemm_bf16_kernel(const __grid_constant__ CUtensorMap tmA0,
                             const __grid_constant__ CUtensorMap tmA1,
                             const __grid_constant__ CUtensorMap tmB, const GemmArgs args) {
  using C = Bf16Cfg<BN, NA, SWIGLU>;
  // rows of the weight tiles: SwiGLU takes rows [mt*128, +128) of gate (A0)
  // and up (A1); the plain store with NA = 2 takes rows [mt*256, +256) of
  // one weight as two halves
  constexpr int kRowStep = SWIGLU ? 128 : 128 * NA;
  constexpr int kRow1 = SWIGLU ? 0 : 128;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kStages * C::kStage);
  uint64_t* empty = full + C::kStages;
  uint64_t* tfull = empty + C::kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint64_t* stallbar = drain + 1;  // test hook: never signalled
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(stallbar + 1);
  volatile uint32_t* abort_flag = tmem_slot + 1;
  volatile uint32_t* consumed = tmem_slot + 2;
  volatile uint32_t* issued = tmem_slot + 3;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < C::kAccBufs; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 4);
    }
    mbar_init(drain, 1);
    mbar_init(stallbar, 1);
    *abort_flag = 0;
    *consumed = 0;
    *issued = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA0);
    if (NA == 2) tma_prefetch_desc(&tmA1);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total_units = total_units_of(args, BN);
  const uint64_t lim = wait_limit(args);

  if (warp == 0 && args.row_token == nullptr) {
    // B rows in a box of the tile's own rows: lane 0 alone waits and loads
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < total_units && ok; u += gridDim.x) {
        const Unit un = decode_unit(u, args, BN);
        for (int kb = 0; kb < args.k_blocks; ++kb, ++it) {
          const int s = it % C::kStages;
          const uint32_t ph = (it / C::kStages) & 1u;
          if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag, lim)) {
            ok = false;
            break;
          }
          uint8_t* st = smem + s * C::kStage;
          mbar_arrive_expect_tx(&full[s], C::kStage);
          tma_load_3d(st, &tmA0, &full[s], kb * 64, un.mt * kRowStep, un.g);
          if (NA == 2)
            tma_load_3d(st + C::kA, &tmA1, &full[s], kb * 64, un.mt * kRowStep + kRow1, un.g);
          tma_load_2d(st + C::kA * C::kNumA, &tmB, &full[s], (kb * 64) % args.b_k, un.row0);
          *issued = it + 1;
        }
      }
      if (!ok) {
        *abort_flag = 1;
        atomicOr(args.status, MOE_DEVICE_WAIT_TIMEOUT);
      }
    }
  } else if (warp == 0) {
    // gathered B rows: lane 0 waits for a free stage and loads the weight
    // tiles, then the lanes load the tile's token rows, four per
    // tile::gather4, lane l taking rows 4l.. and 4(l + 32)..
    uint32_t it = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < total_units && ok; u += gridDim.x) {
      const Unit un = decode_unit(u, args, BN);
      const int n = ((un.nvalid + 15) / 16) * 16;  // rows the MMA reads
      int tok[2][4] = {};
#pragma unroll
      for (int q = 0; q < 2; ++q)
        if (4 * (lane + 32 * q) < n)
          gather_rows(args, un.row0, un.row0 + 4 * (lane + 32 * q), un.row0 + un.nvalid, tok[q]);
      const uint32_t tx = C::kA * C::kNumA + n * 128;
      for (int kb = 0; kb < args.k_blocks; ++kb, ++it) {
        const int s = it % C::kStages;
        const uint32_t ph = (it / C::kStages) & 1u;
        if (lane == 0) ok = mbar_wait(&empty[s], ph ^ 1u, abort_flag, lim);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        uint8_t* st = smem + s * C::kStage;
        if (lane == 0) {
          mbar_arrive_expect_tx(&full[s], tx);
          tma_load_3d(st, &tmA0, &full[s], kb * 64, un.mt * kRowStep, un.g);
          if (NA == 2)
            tma_load_3d(st + C::kA, &tmA1, &full[s], kb * 64, un.mt * kRowStep + kRow1, un.g);
        }
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const int r = 4 * (lane + 32 * q);
          if (r < n)
            tma_gather4(st + C::kA * C::kNumA + r * 128, &tmB, &full[s], kb * 64, tok[q][0],
                        tok[q][1], tok[q][2], tok[q][3]);
        }
        __syncwarp();
        if (lane == 0) *issued = it + 1;
      }
    }
    if (!ok && lane == 0) {
      *abort_flag = 1;
      atomicOr(args.status, MOE_DEVICE_WAIT_TIMEOUT);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      uint32_t it = 0;
      // the test hook's wait on a barrier nothing signals runs out after lim
      bool ok = !args.stall || mbar_wait(stallbar, 0, abort_flag, lim);
      int i = 0;
      for (int u = blockIdx.x; u < total_units && ok; u += gridDim.x, ++i) {
        const Unit un = decode_unit(u, args, BN);
        const int acc = i % C::kAccBufs;
        const int use = i / C::kAccBufs;
        if (!mbar_wait(&tempty[acc], (use & 1) ^ 1, abort_flag, lim)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d0 = tmem_base + acc * C::kAccCols;
        const uint32_t n = static_cast<uint32_t>(((un.nvalid + 15) / 16) * 16);
        const uint32_t idesc = make_idesc(1u, n);
        for (int kb = 0; kb < args.k_blocks; ++kb, ++it) {
          const int s = it % C::kStages;
          const uint32_t ph = (it / C::kStages) & 1u;
          if (!mbar_wait(&full[s], ph, abort_flag, lim)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(smem + s * C::kStage);
          const uint64_t ad0 = sw128_kmajor_desc(a0);
          const uint64_t ad1 = sw128_kmajor_desc(a0 + C::kA);
          const uint64_t bd = sw128_kmajor_desc(a0 + C::kA * C::kNumA);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint32_t accum = (kb | k) ? 1u : 0u;
            // +32 bytes along K inside the swizzled 128-byte row = +2 in addr>>4
            mma_bf16(d0, ad0 + 2 * k, bd + 2 * k, idesc, accum);
            if (NA == 2) mma_bf16(d0 + BN, ad1 + 2 * k, bd + 2 * k, idesc, accum);
          }
          mma_commit(&empty[s]);
          *consumed = it + 1;
        }
        if (!ok) break;
        mma_commit(&tfull[acc]);
      }
      if (!ok) {
        *abort_flag = 1;
        atomicOr(args.status, MOE_DEVICE_WAIT_TIMEOUT);
      }
      // every MMA issued by this thread completes before TMEM is released
      mma_commit(drain);
      mbar_wait(drain, 0, nullptr);
    }
  } else {
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    int i = 0;
    for (int u = blockIdx.x; u < total_units; u += gridDim.x, ++i) {
      const Unit un = decode_unit(u, args, BN);
      const int acc = i % C::kAccBufs;
      const int use = i / C::kAccBufs;
      if (!mbar_wait(&tfull[acc], use & 1, abort_flag, lim)) {
        if (lane == 0) {
          *abort_flag = 1;
          atomicOr(args.status, MOE_DEVICE_WAIT_TIMEOUT);
        }
        break;
      }
      tc_fence_after();
      const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * C::kAccCols;
      const int feat = un.mt * kRowStep + q * 32 + lane;
      for (int c0 = 0; c0 < un.nvalid; c0 += 16) {
        uint32_t g[16], v[16];
        tmem_ld16(tb + c0, g);
        if (NA == 2) tmem_ld16(tb + BN + c0, v);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int col = c0 + j;
          if (col < un.nvalid) {
            const size_t row = static_cast<size_t>(un.row0 + col);
            if (SWIGLU) {
              const float gv = __uint_as_float(g[j]);
              const float uv = __uint_as_float(v[j]);
              const float hv = gv / (1.f + expf(-gv)) * uv;
              static_cast<__nv_bfloat16*>(args.out)[row * args.ld + feat] = __float2bfloat16_rn(hv);
            } else {
              __nv_bfloat16* o = static_cast<__nv_bfloat16*>(args.out) + row * args.ld;
              if (feat < args.m_valid) o[feat] = __float2bfloat16_rn(__uint_as_float(g[j]));
              if (NA == 2 && feat + 128 < args.m_valid)
                o[feat + 128] = __float2bfloat16_rn(__uint_as_float(v[j]));
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (*abort_flag && warp == 0 && lane == 0) {
    // loads issued but never consumed: let them land before the CTA exits
    for (uint32_t j = *consumed; j < *issued; ++j)
      mbar_wait(&full[j % C::kStages], (j / C::kStages) & 1u, nullptr);
  }
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, C::kTmemCols);
}

template <int BN, int NA, bool SWIGLU>
static cudaError_t launch_one(moe_handle* h, const CUtensorMap& a0, const CUtensorMap& a1,
                              const CUtensorMap& b, const GemmArgs& args, cudaStream_t s) {
  using C = Bf16Cfg<BN, NA, SWIGLU>;
  static bool configured[64] = {};  // per device ordinal
  if (h->device < 64 && !configured[h->device]) {
    cudaError_t e = cudaFuncSetAttribute(grouped_gemm_bf16_kernel<BN, NA, SWIGLU>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
    if (e != cudaSuccess) return e;
    configured[h->device] = true;
  }
  grouped_gemm_bf16_kernel<BN, NA, SWIGLU><<<h->num_sms, 192, C::kSmem, s>>>(a0, a1, b, args);
  h->launches++;
  return cudaGetLastError();
}

cudaError_t launch_gemm_bf16(moe_handle* h, bool gated, const GemmPlan& p, cudaStream_t s) {
  const Dims& dm = h->dims;
  GemmArgs a{};
  a.offsets = h->ws.offsets;
  a.unit_base = h->ws.unit_base + (gated ? 0 : (dm.G + 1));
  a.G = dm.G;
  a.m_tiles = p.m_tiles;
  a.k_blocks = p.k_blocks;
  a.bn = p.bn;
  a.status = h->ws.status;
  a.wait_ns = h->fwd_wait_ns;
  a.stall = gated && h->fwd_stall ? 1 : 0;
  a.b_k = gated ? dm.d : dm.f;
  a.m_valid = gated ? dm.f : dm.d;
  const int bi = bn_index(p.bn);
  if (bi < 0) return cudaErrorInvalidValue;
  if (gated) {
    a.out = h->ws.hbuf;
    a.ld = dm.f;
    // short tiles gather their token rows from x; taller ones read the rows
    // the dispatch copied into expert order
    a.row_token = p.gather ? h->ws.row_token : nullptr;
    const CUtensorMap& b = p.gather ? h->tm_xg : h->tm_xp[bi];
    const CUtensorMap &g = h->tm_gate, &u = h->tm_up;
    switch (p.bn) {
      case 16: return launch_one<16, 2, true>(h, g, u, b, a, s);
      case 32: return launch_one<32, 2, true>(h, g, u, b, a, s);
      case 64: return launch_one<64, 2, true>(h, g, u, b, a, s);
      case 96: return launch_one<96, 2, true>(h, g, u, b, a, s);
      case 128: return launch_one<128, 2, true>(h, g, u, b, a, s);
      case 160: return launch_one<160, 2, true>(h, g, u, b, a, s);
      case 192: return launch_one<192, 2, true>(h, g, u, b, a, s);
      case 224: return launch_one<224, 2, true>(h, g, u, b, a, s);
      case 256: return launch_one<256, 2, true>(h, g, u, b, a, s);
      default: return cudaErrorInvalidValue;
    }
  }
  a.out = h->ws.out;
  a.ld = dm.d;
  const CUtensorMap& b = h->tm_h[bi];
  const CUtensorMap& w = h->tm_down;
  if (p.na == 1) {
    // one 128-row weight tile per unit: short tiles, and every tile height
    // when hidden_size is an odd multiple of 128 (no 256-feature units)
    switch (p.bn) {
      case 16: return launch_one<16, 1, false>(h, w, w, b, a, s);
      case 32: return launch_one<32, 1, false>(h, w, w, b, a, s);
      case 64: return launch_one<64, 1, false>(h, w, w, b, a, s);
      case 96: return launch_one<96, 1, false>(h, w, w, b, a, s);
      case 128: return launch_one<128, 1, false>(h, w, w, b, a, s);
      case 160: return launch_one<160, 1, false>(h, w, w, b, a, s);
      case 192: return launch_one<192, 1, false>(h, w, w, b, a, s);
      case 224: return launch_one<224, 1, false>(h, w, w, b, a, s);
      case 256: return launch_one<256, 1, false>(h, w, w, b, a, s);
      default: return cudaErrorInvalidValue;
    }
  }
  switch (p.bn) {
    case 64: return launch_one<64, 2, false>(h, w, w, b, a, s);
    case 96: return launch_one<96, 2, false>(h, w, w, b, a, s);
    case 128: return launch_one<128, 2, false>(h, w, w, b, a, s);
    case 160: return launch_one<160, 2, false>(h, w, w, b, a, s);
    case 192: return launch_one<192, 2, false>(h, w, w, b, a, s);
    case 224: return launch_one<224, 2, false>(h, w, w, b, a, s);
    case 256: return launch_one<256, 2, false>(h, w, w, b, a, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace smoe
