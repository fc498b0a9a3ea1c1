// Grouped expert GEMMs (BF16) on CTA pairs: the same computation as
// gemm_bf16.cu for tall row tiles, with the 2-SM tensor-core MMA.
//
// One tcgen05.mma is issued by one thread, and a thread issues one every
// ~50-80 cycles; an M = 128 MMA with N = 176 rows holds ~88 cycles of tensor
// work, so a single CTA barely keeps its tensor core fed. The pair MMA
// (cta_group::2, M = 256) does twice the work per issued instruction: each
// CTA of a cluster pair holds 128 weight rows and half of the row tile in its
// own shared memory, and each CTA's TMEM receives its 128 rows of the result.
//
// A unit is (expert, 256 output features, row tile). Per CTA pair:
//   producers (warp 0 of each CTA) load that CTA's weight rows (gate and up,
//     or the down projection's) and its half of the row tile; both count
//     their bytes on the even CTA's `full` barrier;
//   the even CTA's warp 1 issues the pair MMAs and commits to the `empty`
//     barriers of both CTAs (and, per unit, to both `tfull` barriers);
//   each CTA's eight epilogue warps (two per TMEM lane quarter, taking
//     alternate 16-column chunks) drain their own TMEM (SwiGLU + BF16 h, or
//     the per-row output, rounded to BF16) and signal the even CTA's `tempty` barrier.
//
// Shared-memory fill from L2, not the tensor core, bounds these kernels at
// prefill sizes (measured: as fast with the MMAs removed), so each unit loads
// only the activation rows its MMA reads: one tensor map per box height (16,
// 32, ..., 128 rows per CTA), picked from the unit's row count. When the
// gated accumulators fill TMEM (row tiles over 128, one buffer), the epilogue
// computes h into packed BF16 registers, releases TMEM, and only then stores,
// so the next unit's MMAs overlap the global stores.
// Gate/up units are handed out dynamically (~55 long units per pair whose
// cost varies with the row count): the even CTA's producer takes the next
// unit index from a per-launch counter in global memory and publishes it
// through a small ring in both CTAs' shared memory; the MMA thread, both
// CTAs' epilogue warps and the odd CTA's producer read it from there and
// release the slot. An index past the last unit ends every role's loop.
// Down-projection units are short and many (~195 per pair, balanced by their
// number): there every role walks the static sequence pair, pair + pairs, ...
// (measured: the publication's cross-CTA latency at each unit start costs the
// down GEMM more than dynamic balance gains).
// Every wait is bounded as in gemm_bf16.cu. The only unbounded step is the
// cluster barrier at entry and exit, which both CTAs always reach.
#include <cuda_bf16.h>
#include <stdio.h>

#include "gemm_common.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace smoe {

using namespace sm100;

constexpr int kPairBoxes = 8;     // activation box heights 16, 32, ..., 128 rows
constexpr int kPairEpiWarps = 8;  // two per TMEM lane quarter
constexpr int kUnitRing = 8;      // unit indices published ahead of the slowest reader
// readers of each published unit index: the MMA thread, the epilogue warps of
// both CTAs and the odd CTA's producer
constexpr int kUnitReaders = 2 + 2 * kPairEpiWarps;
constexpr int kPairThreads = 64 + 32 * kPairEpiWarps;
// The register file is four 16K-register slices, one per SM sub-partition,
// and warp w runs on slice w % 4: ten warps put three on a slice.
constexpr int kPairRegs = 16384 / (32 * ((kPairThreads / 32 + 3) / 4)) / 8 * 8;

struct PairBoxMaps {
  CUtensorMap m[kPairBoxes];  // m[i]: box of 16 * (i + 1) rows x 64 columns
};

template <int BN, bool SWIGLU>
struct Pair2Cfg {
  static constexpr int kA = 128 * 64 * 2;        // this CTA's 128 x 64 BF16 weight tile
  static constexpr int kB = (BN / 2) * 64 * 2;   // this CTA's half of the row tile
  static constexpr int kNumA = SWIGLU ? 2 : 1;
  // 64-column K blocks per stage: two for the down projection, so that every
  // stage carries eight MMAs like the gate/up stage (a stage's barrier round
  // trip costs ~600 cycles, which four MMAs of a short row tile do not cover)
  static constexpr int kKSub = SWIGLU ? 1 : 2;
  static constexpr int kABytes = kA * kNumA * kKSub;
  static constexpr int kStage = kABytes + kB * kKSub;
  static constexpr int kStages0 = (227 * 1024 - 2048) / kStage;
  static constexpr int kStages = kStages0 > 12 ? 12 : kStages0;
  static constexpr int kAccCols = kNumA * BN;
  static constexpr int kAccBufs = 2 * kAccCols <= 512 ? 2 : 1;
  static constexpr int kTmemCols = pow2_at_least(kAccBufs * kAccCols, 32);
  static constexpr int kSmem = kStages * kStage + 1024 + 512;
  static_assert(BN % 32 == 0, "each CTA's half of the row tile is a multiple of 16 rows");
  static_assert(kStage % 1024 == 0, "stage must keep 1024-byte alignment");
  static_assert(kTmemCols <= 512, "TMEM holds 512 columns");
  static_assert(kStages >= 2, "need at least two stages");
  static_assert(BN / 2 <= 16 * kPairBoxes, "a box per half row tile");
  // gated tiles that fill TMEM drain into registers first (two BF16 per
  // register, half of the 16-column chunks per warp)
  static constexpr bool kDrainFirst = SWIGLU && kAccBufs == 1;
  static constexpr int kChunksPerWarp = BN / 32;
};

// silu(g) * u with IEEE expf and division, the same arithmetic as the 1-SM
// and FP8 kernels, so a token's h does not depend on which kernel its batch
// size selects.
__device__ __forceinline__ float silu_mul(float g, float u) {
  return g / (1.f + expf(-g)) * u;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

template <int BN, bool SWIGLU>
__global__ void __maxnreg__(kPairRegs)
    grouped_gemm_bf16_pair_kernel(const __grid_constant__ CUtensorMap tmA0,
                                  const __grid_constant__ CUtensorMap tmA1,
                                  const __grid_constant__ PairBoxMaps tmB, const GemmArgs args) {
  using C = Pair2Cfg<BN, SWIGLU>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kStages * C::kStage);
  uint64_t* empty = full + C::kStages;
  uint64_t* tfull = empty + C::kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint64_t* stallbar = drain + 1;          // test hook: never signalled
  uint64_t* uq_full = stallbar + 1;        // [kUnitRing] a unit index was published
  uint64_t* uq_empty = uq_full + kUnitRing;  // [kUnitRing] (even CTA) every reader has it
  int32_t* uq = reinterpret_cast<int32_t*>(uq_empty + kUnitRing);  // [kUnitRing]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(uq + kUnitRing);
  volatile uint32_t* abort_flag = tmem_slot + 1;
  volatile uint32_t* consumed = tmem_slot + 2;
  volatile uint32_t* issued = tmem_slot + 3;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0: issues the MMAs
  const bool dynamic = args.sched != nullptr;
  const int pair = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < C::kAccBufs; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 2 * kPairEpiWarps);  // the epilogue warps of both CTAs
    }
    mbar_init(drain, 1);
    mbar_init(stallbar, 1);
    for (int j = 0; j < kUnitRing; ++j) {
      mbar_init(&uq_full[j], 1);
      mbar_init(&uq_empty[j], kUnitReaders);
    }
    *abort_flag = 0;
    *consumed = 0;
    *issued = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 0) {
    if (lane == 0) tma_prefetch_desc(&tmA0);
    if (SWIGLU && lane == 1) tma_prefetch_desc(&tmA1);
    if (lane >= 2 && lane - 2 < BN / 32) tma_prefetch_desc(&tmB.m[lane - 2]);
  }
  cluster_sync();  // the peer's barriers exist before anything signals them
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, C::kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();  // both CTAs' TMEM is allocated before the first pair MMA
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total_units = total_units_of(args, BN);
  const uint64_t lim = wait_limit(args);
  // j-th unit index of this pair (every reader; false: a wait gave up)
  auto read_unit = [&](uint32_t j, int* u) -> bool {
    if (!dynamic) {
      *u = pair + static_cast<int>(j) * npairs;
      return true;
    }
    const int slot = static_cast<int>(j % kUnitRing);
    const uint32_t ph = (j / kUnitRing) & 1u;
    const bool ok = rank == 0 ? mbar_wait(&uq_full[slot], ph, abort_flag, lim)
                              : mbar_wait_cluster(&uq_full[slot], ph, abort_flag, lim);
    if (!ok) return false;
    *u = uq[slot];
    return true;
  };
  auto release_unit = [&](uint32_t j) {
    if (!dynamic) return;
    const int slot = static_cast<int>(j % kUnitRing);
    if (rank == 0) mbar_arrive(&uq_empty[slot]);
    else mbar_arrive_remote(&uq_empty[slot], 0);
  };

  if (warp == 0) {
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      // the even CTA takes unit indices one ahead, so the atomic's round trip
      // overlaps the current unit's loads
      int next_u = dynamic && rank == 0 ? atomicAdd(args.sched, 1) : 0;
      for (uint32_t j = 0; ok; ++j) {
        int u;
        if (dynamic && rank == 0) {
          // publish the next unit to both CTAs
          const int slot = static_cast<int>(j % kUnitRing);
          if (!mbar_wait_cluster(&uq_empty[slot], ((j / kUnitRing) & 1u) ^ 1u, abort_flag, lim)) {
            ok = false;
            break;
          }
          u = next_u;
          if (u < total_units) next_u = atomicAdd(args.sched, 1);
          uq[slot] = u;
          st_shared_remote_u32(&uq[slot], 1, static_cast<uint32_t>(u));
          mbar_arrive(&uq_full[slot]);
          mbar_arrive_remote(&uq_full[slot], 1);
        } else {
          if (!read_unit(j, &u)) {
            ok = false;
            break;
          }
          release_unit(j);
        }
        if (u >= total_units) break;
        const Unit un = decode_unit(u, args, BN);
        const int n = ((un.nvalid + 31) / 32) * 32;  // MMA N: halves of 16-row multiples
        const int arow = un.mt * 256 + static_cast<int>(rank) * 128;
        const int brow = un.row0 + static_cast<int>(rank) * (n / 2);
        const CUtensorMap* bmap = &tmB.m[n / 32 - 1];  // box of n / 2 rows
        const uint32_t tx = 2u * static_cast<uint32_t>(C::kABytes + C::kKSub * (n / 2) * 128);
        for (int ks = 0; ks < args.k_blocks / C::kKSub; ++ks, ++it) {
          const int s = it % C::kStages;
          const uint32_t ph = (it / C::kStages) & 1u;
          if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag, lim)) {
            ok = false;
            break;
          }
          uint8_t* st = smem + s * C::kStage;
          if (rank == 0) mbar_arrive_expect_tx(&full[s], tx);
#pragma unroll
          for (int sub = 0; sub < C::kKSub; ++sub) {
            const int kc = (ks * C::kKSub + sub) * 64;
            uint8_t* a = st + sub * C::kNumA * C::kA;
            tma_load_3d_pair(a, &tmA0, &full[s], kc, arow, un.g);
            if (SWIGLU) tma_load_3d_pair(a + C::kA, &tmA1, &full[s], kc, arow, un.g);
            tma_load_2d_pair(st + C::kABytes + sub * C::kB, bmap, &full[s], kc, brow);
          }
          *issued = it + 1;
        }
      }
      if (!ok) {
        *abort_flag = 1;
        atomicOr(args.status, MOE_DEVICE_WAIT_TIMEOUT);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      uint32_t it = 0;
      // the test hook's wait on a barrier nothing signals runs out after lim
      bool ok = !args.stall || mbar_wait(stallbar, 0, abort_flag, lim);
      for (uint32_t i = 0; ok; ++i) {
        int u;
        if (!read_unit(i, &u)) {
          ok = false;
          break;
        }
        release_unit(i);
        if (u >= total_units) break;
        const Unit un = decode_unit(u, args, BN);
        const int acc = i % C::kAccBufs;
        const int use = i / C::kAccBufs;
        if (!mbar_wait(&tempty[acc], (use & 1) ^ 1, abort_flag, lim)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d0 = tmem_base + acc * C::kAccCols;
        const uint32_t n = static_cast<uint32_t>(((un.nvalid + 31) / 32) * 32);
        const uint32_t idesc = make_idesc(1u, n, 256);
        for (int ks = 0; ks < args.k_blocks / C::kKSub; ++ks, ++it) {
          const int s = it % C::kStages;
          const uint32_t ph = (it / C::kStages) & 1u;
          if (!mbar_wait(&full[s], ph, abort_flag, lim)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(smem + s * C::kStage);
#pragma unroll
          for (int sub = 0; sub < C::kKSub; ++sub) {
            const uint64_t ad0 = sw128_kmajor_desc(a0 + sub * C::kNumA * C::kA);
            const uint64_t ad1 = sw128_kmajor_desc(a0 + sub * C::kNumA * C::kA + C::kA);
            const uint64_t bd = sw128_kmajor_desc(a0 + C::kABytes + sub * C::kB);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const uint32_t accum = (ks | sub | k) ? 1u : 0u;
              mma_bf16_pair(d0, ad0 + 2 * k, bd + 2 * k, idesc, accum);
              if (SWIGLU) mma_bf16_pair(d0 + BN, ad1 + 2 * k, bd + 2 * k, idesc, accum);
            }
          }
          mma_commit_pair(&empty[s], 0x3);
          *consumed = it + 1;
        }
        if (!ok) break;
        mma_commit_pair(&tfull[acc], 0x3);
      }
      if (!ok) {
        *abort_flag = 1;
        atomicOr(args.status, MOE_DEVICE_WAIT_TIMEOUT);
      }
      mma_commit_pair(drain, 0x1);  // this CTA only
      mbar_wait(drain, 0, nullptr);
    }
  } else {
    const int q = warp & 3;           // TMEM lane quarter this warp may access
    const int half = (warp - 2) >> 2;  // which alternate 16-column chunks
    for (uint32_t i = 0;; ++i) {
      int u;
      if (!read_unit(i, &u)) {
        if (lane == 0) {
          *abort_flag = 1;
          atomicOr(args.status, MOE_DEVICE_WAIT_TIMEOUT);
        }
        break;
      }
      __syncwarp();
      if (lane == 0) release_unit(i);
      if (u >= total_units) break;
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
      const int feat = un.mt * 256 + static_cast<int>(rank) * 128 + q * 32 + lane;
      if constexpr (C::kDrainFirst) {
        uint32_t hp[C::kChunksPerWarp * 8];
#pragma unroll
        for (int j = 0; j < C::kChunksPerWarp; ++j) {
          const int c0 = (2 * j + half) * 16;
          if (c0 < un.nvalid) {
            uint32_t g[16], v[16];
            tmem_ld16(tb + c0, g);
            tmem_ld16(tb + BN + c0, v);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 8; ++e)
              hp[j * 8 + e] =
                  pack_bf16x2(silu_mul(__uint_as_float(g[2 * e]), __uint_as_float(v[2 * e])),
                              silu_mul(__uint_as_float(g[2 * e + 1]), __uint_as_float(v[2 * e + 1])));
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (rank == 0) mbar_arrive(&tempty[acc]);
          else mbar_arrive_remote(&tempty[acc], 0);
        }
        uint16_t* out = static_cast<uint16_t*>(args.out);
#pragma unroll
        for (int j = 0; j < C::kChunksPerWarp; ++j) {
          const int c0 = (2 * j + half) * 16;
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int col = c0 + e;
            if (col < un.nvalid) {
              const uint32_t w = hp[j * 8 + e / 2];
              out[static_cast<size_t>(un.row0 + col) * args.ld + feat] =
                  static_cast<uint16_t>((e & 1) ? (w >> 16) : (w & 0xFFFFu));
            }
          }
        }
      } else {
        for (int c0 = half * 16; c0 < un.nvalid; c0 += 32) {
          uint32_t g[16], v[16];
          tmem_ld16(tb + c0, g);
          if (SWIGLU) tmem_ld16(tb + BN + c0, v);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int col = c0 + j;
            if (col < un.nvalid) {
              const size_t row = static_cast<size_t>(un.row0 + col);
              if (SWIGLU) {
                const float hv = silu_mul(__uint_as_float(g[j]), __uint_as_float(v[j]));
                static_cast<__nv_bfloat16*>(args.out)[row * args.ld + feat] = __float2bfloat16_rn(hv);
              } else if (feat < args.m_valid) {
                static_cast<__nv_bfloat16*>(args.out)[row * args.ld + feat] =
                    __float2bfloat16_rn(__uint_as_float(g[j]));
              }
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (rank == 0) mbar_arrive(&tempty[acc]);
          else mbar_arrive_remote(&tempty[acc], 0);
        }
      }
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (*abort_flag && rank == 0 && warp == 0 && lane == 0) {
    // loads counted on this CTA's full barriers (both CTAs') that were never
    // consumed: let them land before either CTA exits
    for (uint32_t j = *consumed; j < *issued; ++j)
      mbar_wait(&full[j % C::kStages], (j / C::kStages) & 1u, nullptr);
  }
  cluster_sync();
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem_base, C::kTmemCols);
}

template <int BN, bool SWIGLU>
static cudaError_t launch_pair(moe_handle* h, const CUtensorMap& a0, const CUtensorMap& a1,
                               const PairBoxMaps& b, const GemmArgs& args, cudaStream_t s) {
  using C = Pair2Cfg<BN, SWIGLU>;
  auto kern = grouped_gemm_bf16_pair_kernel<BN, SWIGLU>;
  static bool configured[64] = {};
  if (h->device < 64 && !configured[h->device]) {
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
    if (e != cudaSuccess) return e;
    configured[h->device] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(h->num_sms & ~1));
  cfg.blockDim = dim3(kPairThreads);
  cfg.dynamicSmemBytes = C::kSmem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, a0, a1, b, args);
  h->launches++;
  return e != cudaSuccess ? e : cudaGetLastError();
}

// The pair kernel's row-tile heights (multiples of 32, each CTA taking half).
bool pair_bn_supported(int bn) {
  return bn == 128 || bn == 160 || bn == 192 || bn == 224 || bn == 256;
}

cudaError_t launch_gemm_bf16_pair(moe_handle* h, bool gated, const GemmPlan& p, cudaStream_t s) {
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
  a.sched = gated ? h->ws.sched : nullptr;  // dynamic units for gate/up only
  // activation maps with boxes of 16, 32, ..., 128 rows (each CTA's half of
  // a row tile of 32, 64, ..., 256)
  PairBoxMaps b;
  for (int i = 0; i < kPairBoxes; ++i) b.m[i] = (gated ? h->tm_xp : h->tm_h)[bn_index(16 * (i + 1))];
  if (gated) {
    a.out = h->ws.hbuf;
    a.ld = dm.f;
    const CUtensorMap &g = h->tm_gate, &u = h->tm_up;
    switch (p.bn) {
      case 128: return launch_pair<128, true>(h, g, u, b, a, s);
      case 160: return launch_pair<160, true>(h, g, u, b, a, s);
      case 192: return launch_pair<192, true>(h, g, u, b, a, s);
      case 224: return launch_pair<224, true>(h, g, u, b, a, s);
      case 256: return launch_pair<256, true>(h, g, u, b, a, s);
      default: return cudaErrorInvalidValue;
    }
  }
  a.out = h->ws.out;
  a.ld = dm.d;
  const CUtensorMap& w = h->tm_down;
  switch (p.bn) {
    case 128: return launch_pair<128, false>(h, w, w, b, a, s);
    case 160: return launch_pair<160, false>(h, w, w, b, a, s);
    case 192: return launch_pair<192, false>(h, w, w, b, a, s);
    case 224: return launch_pair<224, false>(h, w, w, b, a, s);
    case 256: return launch_pair<256, false>(h, w, w, b, a, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace smoe
