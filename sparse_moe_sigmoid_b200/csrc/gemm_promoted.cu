// Grouped expert GEMMs for e4m3 weights with one fp32 scale per 128x128 block
// and dynamically quantised e4m3 activations (one fp32 scale per row per 128
// columns).
//
// Weight format: "Kimi K2 · Down projection" (OpenModelAtlas), the
// config.json quantization_config excerpt (fmt e4m3, weight_block_size
// [128, 128], activation_scheme dynamic) and the note that every 128 x 128
// block carries one scale. With W = q_w * s_w and x = q_x * s_x per block,
//   (W x)[n] = sum_kb  s_w[n/128, kb] * s_x[kb] * sum_{k in kb} q_w[n,k] q_x[k]
// The inner sum is an e4m3 x e4m3 tensor-core MMA (tcgen05 kind::f8f6f4,
// K = 32 per instruction, 4 per 128-column block) into an fp32 partial in
// TMEM; the scales differ per block, so each block's partial is promoted
// separately: four promotion warps read it (tcgen05.ld), multiply by
// s_w * s_x[row] and add into fp32 registers. The partial rotates through up
// to four TMEM buffers, so the MMAs of the next blocks run while block kb is
// promoted. (The hardware's own block scaling takes power-of-two ue8m0
// scales per 32 columns; the K2 scales are arbitrary fp32 per 128, so it does
// not apply.)
//
// Gate/up epilogue: h = silu(g) * u in fp32, then h is quantised per row per
// 128 features, which is exactly this tile's 128 features: s_h = amax/448,
// q = e4m3(h / s_h) (correctly rounded divisions, nearest-even saturating
// conversion), written with its scale for the down GEMM.
// Down epilogue: the promoted fp32 row outputs, rounded to BF16 once.
//
// The same kernel with BF16 operands and no scales computes the router
// logits on the tensor cores (launch_router_gemm below): there the point of
// promoting every 128 K is precision, not scaling. The tensor core adds each
// MMA's products into its fp32 accumulator with a rounding that, over
// K = 3 x 7168, drifts by more than the 1e-5 band in which the top-k choice
// may legitimately differ; partial sums over 128 K stay small (so their
// rounding is tiny) and are added in fp32 registers with round-to-nearest.
//
// Roles and the bounded-wait / wind-down rules are those of the BF16 kernel
// (gemm_bf16.cu): warp 0 TMA producer, warp 1 TMEM owner and MMA issuer,
// then NPG warpgroups of promotion + epilogue warps; group g owns columns
// [g*BN/NPG, (g+1)*BN/NPG) of the row tile (two groups halve the promotion
// work per thread and allow tiles of 128 rows with gate and up, 256 without).
// The shared-memory ring's depth is set at launch from what the scale
// staging of the actual K leaves free.
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <stdio.h>

#include "gemm_common.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace smoe {

using namespace sm100;

// promotion warpgroups of the 64-row FP8 gate/up tile (a tuning constant:
// two hold 32 columns a thread, four hold 16 with fewer registers each;
// four measured no faster where 64-row tiles run)
#ifndef SMOE_FP8_GU64_NPG
#define SMOE_FP8_GU64_NPG 2
#endif
constexpr int kFp8MaxKBlocks = 64;  // hidden_size and moe_intermediate_size <= 8192
constexpr int kPromMaxStages = 12;
constexpr int kPromSmemBudget = 227 * 1024 - 2048;

// FP8: e4m3 operands, 128 K per stage, block scales applied at promotion.
// Otherwise BF16 operands, 64 K per stage, no scales.
// DUAL (FP8 down projection, short row tiles): two consecutive 128-feature
// weight tiles per unit, loaded, multiplied and promoted like gate and up,
// both stored as row outputs, so that a stage carries two weight tiles.
template <int BN, bool GATED, bool FP8, int NPG, bool DUAL = false>
struct PromCfg {
  static constexpr bool kTwoA = GATED || DUAL;
  static constexpr int kThreads = 64 + 128 * NPG;
  static constexpr int kCols = BN / NPG;  // columns per promotion group
  static constexpr int kBatch = NPG >= 3 ? 16 : kCols;  // TMEM columns per load batch
  static constexpr int kA = 128 * 128;    // 128 rows x 128 bytes of K
  static constexpr int kB = BN * 128;
  static constexpr int kKPerStage = FP8 ? 128 : 64;
  static constexpr int kNumA = kTwoA ? 2 : 1;
  static constexpr int kStage = kA * kNumA + kB;
  static constexpr int kAmaxBytes = GATED ? 4 * BN * 4 : 0;
  static constexpr int kPCols = kTwoA ? 2 * BN : BN;  // one partial buffer
  // partial buffers in TMEM: as many as fit (up to 4), so that the MMAs can
  // run several blocks ahead of the promotion (a hand-over costs an MMA
  // completion plus two mbarrier wake-ups, several hundred cycles)
  static constexpr int kPBufs = 512 / pow2_at_least(kPCols, 32) >= 4   ? 4
                                : 512 / pow2_at_least(kPCols, 32) >= 2 ? 2
                                                                       : 1;
  static constexpr int kTmemCols = pow2_at_least(kPBufs * kPCols, 32);
  static constexpr int kBarrierBytes = 512;
  static_assert(kStage % 1024 == 0, "stage must keep 1024-byte alignment");
  static_assert(kCols % 16 == 0, "columns per group in 16-column loads");
  static_assert((kTwoA ? 2 : 1) * kCols <= 64, "one promotion's loads must fit in registers");
  static_assert(!(GATED && DUAL) && (FP8 || !DUAL), "DUAL is the plain FP8 mode");
  static_assert(kTmemCols <= 512, "TMEM holds 512 columns");
  static_assert(kPBufs >= 2, "the promotion needs two partial buffers at least");
  static_assert(FP8 || !GATED, "the BF16 promoted GEMM is plain");
  static_assert(!GATED || BN <= 128, "a gathered tile takes at most one gather4 per lane");
  // Tall tiles (three promotion warpgroups, the promotion-bound regime) stage
  // the products s_w * s_x per block and row, once per tile, so the promotion
  // does one multiply-add per value; the others stage s_x and s_w and
  // multiply per value (one stage more of the ring at mid sizes).
  static constexpr bool kPreMul = FP8 && NPG >= 3;
  // scale staging of FP8: [KB][BN] activation scales (or products, one array
  // per weight tile) and [2][KB] weight scales
  static constexpr int scale_bytes(int kb) {
    return !FP8 ? 0 : kPreMul ? (kTwoA ? 2 : 1) * kb * BN * 4 : (kb * BN + 2 * kb) * 4;
  }
  // Tall FP8 tiles (three promotion warpgroups) leave 44 KB of the SM's
  // shared memory to L1, one ring stage fewer: the per-tile scale staging and
  // the unit decoding read through it. Measured at T = 16384 in two runs:
  // gate/up (96-row tiles, 4 -> 3 stages) 11.6-11.8 -> 11.1-11.2 ms, down
  // (192-row tiles, 5 -> 4 stages) 6.5-6.6 -> 6.3 ms; T = 4096 3.90 -> 3.76 ms
  // (gate/up); unchanged at T = 1024.
  static constexpr int kL1Reserve = FP8 && NPG >= 3 ? 45056 : 0;
  static constexpr int stages(int kb) {
    const int n =
        (kPromSmemBudget - kL1Reserve - kBarrierBytes - scale_bytes(kb) - kAmaxBytes) / kStage;
    return n > kPromMaxStages ? kPromMaxStages : n;
  }
  static constexpr int smem(int kb) {
    return stages(kb) * kStage + scale_bytes(kb) + kAmaxBytes + kBarrierBytes + 1024;
  }
};

// Two fp32 operations per instruction (sm_100 packed fp32): the same IEEE
// round-to-nearest results as two scalar ones. The promotion's arithmetic is
// the FP8 GEMMs' critical path at large T (measured: ~1000 cycles per 128-K
// block against ~400 of MMA work).
__device__ __forceinline__ void fma2(float& a0, float& a1, float x0, float x1, float c0,
                                     float c1) {
  asm("{\n\t.reg .b64 A, X, C;\n\t"
      "mov.b64 A, {%0, %1};\n\tmov.b64 X, {%2, %3};\n\tmov.b64 C, {%4, %5};\n\t"
      "fma.rn.f32x2 A, X, C, A;\n\tmov.b64 {%0, %1}, A;\n\t}"
      : "+f"(a0), "+f"(a1)
      : "f"(x0), "f"(x1), "f"(c0), "f"(c1));
}

__device__ __forceinline__ void mul2(float& d0, float& d1, float x0, float x1, float y0, float y1) {
  asm("{\n\t.reg .b64 D, X, Y;\n\t"
      "mov.b64 X, {%2, %3};\n\tmov.b64 Y, {%4, %5};\n\t"
      "mul.rn.f32x2 D, X, Y;\n\tmov.b64 {%0, %1}, D;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(x0), "f"(x1), "f"(y0), "f"(y1));
}

// registers per thread for the one CTA per SM: the register file is four
// 16K-register slices, one per scheduler, and a block's warps are spread over
// them, so a slice holds ceil(warps / 4) warps; rounded down to the
// allocation granule of 8, at most 255
template <int kThreads>
constexpr int prom_max_regs() {
  return (16384 / (32 * ((kThreads / 32 + 3) / 4))) / 8 * 8 > 255
             ? 255
             : (16384 / (32 * ((kThreads / 32 + 3) / 4))) / 8 * 8;
}

template <int NPG>
constexpr int prom_regs() {
  return prom_max_regs<64 + 128 * NPG>();
}

template <int BN, bool GATED, bool FP8, int NPG, bool DUAL>
__global__ void __maxnreg__(prom_regs<NPG>())
    grouped_gemm_promoted_kernel(const __grid_constant__ CUtensorMap tmA0,
                                 const __grid_constant__ CUtensorMap tmA1,
                                 const __grid_constant__ CUtensorMap tmB, const GemmArgs args) {
  using C = PromCfg<BN, GATED, FP8, NPG, DUAL>;
  const int KB = args.k_blocks / (args.ksplit > 1 ? args.ksplit : 1);  // k-blocks per unit
  const int S = args.stages;  // ring depth, set at launch (<= kPromMaxStages)
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  float* sa_s = reinterpret_cast<float*>(smem + S * C::kStage);  // [KB][BN] (FP8)
  // kPreMul: sa_s holds s_w0 * s_x and sb_s s_w1 * s_x; else sw_s the s_w
  float* sb_s = sa_s + (C::kPreMul && C::kTwoA ? KB * BN : 0);
  float* sw_s = sa_s + (FP8 ? (C::kPreMul ? (C::kTwoA ? 2 : 1) * KB * BN : KB * BN) : 0);
  float* amax_s = sw_s + (FP8 && !C::kPreMul ? 2 * KB : 0);       // [4][BN] (gated)
  uint64_t* full = reinterpret_cast<uint64_t*>(
      (reinterpret_cast<uintptr_t>(amax_s + (GATED ? 4 * BN : 0)) + 7) & ~uintptr_t(7));
  uint64_t* empty = full + kPromMaxStages;
  uint64_t* pfull = empty + kPromMaxStages;
  uint64_t* pempty = pfull + 4;
  uint64_t* drain = pempty + 4;
  uint64_t* grp = drain + 1;  // the promotion threads' own barrier (bounded waits)
  uint64_t* stallbar = grp + 1;  // test hook: never signalled
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(stallbar + 1);
  volatile uint32_t* abort_flag = tmem_slot + 1;
  volatile uint32_t* consumed = tmem_slot + 2;
  volatile uint32_t* issued = tmem_slot + 3;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // stages accumulated in TMEM per promotion (FP8: every block, its scales
  // differ); the router's K slices after the first use kpp_rest
  auto kpp_of = [&](const Unit& un) {
    return FP8 ? 1 : (un.split > 0 && args.kpp_rest > 0 ? args.kpp_rest : args.kpp);
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < C::kPBufs; ++a) {
      mbar_init(&pfull[a], 1);
      mbar_init(&pempty[a], 4 * NPG);
    }
    mbar_init(drain, 1);
    mbar_init(grp, 128 * NPG);
    mbar_init(stallbar, 1);
    *abort_flag = 0;
    *consumed = 0;
    *issued = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA0);
    if (C::kTwoA) tma_prefetch_desc(&tmA1);
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
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % S;
          const uint32_t ph = (it / S) & 1u;
          if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag, lim)) {
            ok = false;
            break;
          }
          uint8_t* st = smem + s * C::kStage;
          mbar_arrive_expect_tx(&full[s], C::kStage);
          const int kc = (un.split * KB + kb) * C::kKPerStage;
          const int arow = DUAL ? un.mt * 256 : un.mt * 128;
          tma_load_3d(st, &tmA0, &full[s], kc, arow, un.g);
          if (C::kTwoA) tma_load_3d(st + C::kA, &tmA1, &full[s], kc, arow + (DUAL ? 128 : 0), un.g);
          tma_load_2d(st + C::kA * C::kNumA, &tmB, &full[s], kc % args.b_k, un.row0);
          *issued = it + 1;
        }
      }
      if (!ok) {
        *abort_flag = 1;
        atomicOr(args.status, MOE_DEVICE_WAIT_TIMEOUT);
      }
    }
  } else if (warp == 0) {
    // gathered B rows (gate/up): lane 0 waits for a free stage and loads the
    // weight tiles, then the lanes load the tile's token rows, four per
    // tile::gather4 (at most 128 rows: one gather per lane)
    uint32_t it = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < total_units && ok; u += gridDim.x) {
      const Unit un = decode_unit(u, args, BN);
      const int n = ((un.nvalid + 15) / 16) * 16;  // rows the MMA reads
      int tok[4] = {};
      if (4 * lane < n) gather_rows(args, un.row0, un.row0 + 4 * lane, un.row0 + un.nvalid, tok);
      const uint32_t tx = C::kA * C::kNumA + n * 128;
      for (int kb = 0; kb < KB; ++kb, ++it) {
        const int s = it % S;
        const uint32_t ph = (it / S) & 1u;
        if (lane == 0) ok = mbar_wait(&empty[s], ph ^ 1u, abort_flag, lim);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        uint8_t* st = smem + s * C::kStage;
        const int kc = (un.split * KB + kb) * C::kKPerStage;
        if (lane == 0) {
          mbar_arrive_expect_tx(&full[s], tx);
          const int arow = DUAL ? un.mt * 256 : un.mt * 128;
          tma_load_3d(st, &tmA0, &full[s], kc, arow, un.g);
          if (C::kTwoA)
            tma_load_3d(st + C::kA, &tmA1, &full[s], kc, arow + (DUAL ? 128 : 0), un.g);
        }
        if (4 * lane < n)
          tma_gather4(st + C::kA * C::kNumA + 4 * lane * 128, &tmB, &full[s], kc % args.b_k,
                      tok[0], tok[1], tok[2], tok[3]);
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
      uint32_t it = 0;   // stages consumed so far
      uint32_t pit = 0;  // promotions handed over so far (the partial-buffer sequence)
      // the test hook's wait on a barrier nothing signals runs out after lim
      bool ok = !args.stall || mbar_wait(stallbar, 0, abort_flag, lim);
      for (int u = blockIdx.x; u < total_units && ok; u += gridDim.x) {
        const Unit un = decode_unit(u, args, BN);
        const uint32_t n = static_cast<uint32_t>(((un.nvalid + 15) / 16) * 16);
        const uint32_t idesc = make_idesc(FP8 ? 0u : 1u, n);
        const int KPP = kpp_of(un);
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % S;
          const uint32_t ph = (it / S) & 1u;
          const int pb = pit % C::kPBufs;
          const int sub = kb % KPP;
          if ((sub == 0 &&
               !mbar_wait(&pempty[pb], ((pit / C::kPBufs) & 1u) ^ 1u, abort_flag, lim)) ||
              !mbar_wait(&full[s], ph, abort_flag, lim)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(smem + s * C::kStage);
          const uint64_t ad0 = sw128_kmajor_desc(a0);
          const uint64_t ad1 = sw128_kmajor_desc(a0 + C::kA);
          const uint64_t bd = sw128_kmajor_desc(a0 + C::kA * C::kNumA);
          const uint32_t d0 = tmem_base + pb * C::kPCols;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint32_t accum = (k | sub) ? 1u : 0u;  // each promotion's partial starts fresh
            if (FP8) {
              mma_fp8(d0, ad0 + 2 * k, bd + 2 * k, idesc, accum);
              if (C::kTwoA) mma_fp8(d0 + BN, ad1 + 2 * k, bd + 2 * k, idesc, accum);
            } else {
              mma_bf16(d0, ad0 + 2 * k, bd + 2 * k, idesc, accum);
            }
          }
          mma_commit(&empty[s]);
          if (sub == KPP - 1 || kb == KB - 1) {
            mma_commit(&pfull[pb]);
            ++pit;
          }
          *consumed = it + 1;
        }
      }
      if (!ok) {
        *abort_flag = 1;
        atomicOr(args.status, MOE_DEVICE_WAIT_TIMEOUT);
      }
      mma_commit(drain);
      mbar_wait(drain, 0, nullptr);
    }
  } else {
    const int q = warp & 3;                    // TMEM lane quarter
    const int ptid = threadIdx.x - 64;         // 0 .. 128*NPG-1 among the promotion warps
    const int c_begin = (ptid >> 7) * C::kCols;  // this group's first column
    uint32_t pit = 0, gph = 0;
    bool ok = true;
    auto group_sync = [&]() {
      mbar_arrive(grp);
      const bool r = mbar_wait(grp, gph, abort_flag, lim);
      gph ^= 1u;
      return r;
    };
    for (int u = blockIdx.x; u < total_units && ok; u += gridDim.x) {
      const Unit un = decode_unit(u, args, BN);
      const int KPP = kpp_of(un);
      const int NP = (KB + KPP - 1) / KPP;  // promotions of this tile
      if (FP8) {
        // this tile's scales: activations [KB][BN] and the weight block scales
        if (!group_sync()) {  // the previous tile's readers are done
          ok = false;
          break;
        }
        // weight block scales [G][rows / 128][KB]: the tile's row of blocks
        // (DUAL: the two consecutive rows of its two tiles)
        const size_t wrow = DUAL ? ((size_t)un.g * 2 * args.m_tiles + 2 * un.mt) * KB
                                 : ((size_t)un.g * args.m_tiles + un.mt) * KB;
        const float* ws1 = GATED ? args.w_scale1 + wrow : args.w_scale0 + wrow + KB;
        for (int i = ptid; i < KB * BN; i += 128 * NPG) {
          const int kb = i / BN, j = i - kb * BN;
          // the scales of the B row: the token's (gathered x) or the row's own (h)
          const int r = j < un.nvalid ? (args.row_token ? __ldg(args.row_token + un.row0 + j)
                                                         : un.row0 + j)
                                      : -1;
          const float sx = r >= 0 ? __ldg(args.act_scale + (size_t)r * KB + kb) : 0.f;
          if (C::kPreMul) {  // the products the promotion multiplies by
            sa_s[i] = __ldg(args.w_scale0 + wrow + kb) * sx;
            if (C::kTwoA) sb_s[i] = __ldg(ws1 + kb) * sx;
          } else {
            sa_s[i] = sx;
          }
        }
        if (!C::kPreMul) {
          for (int i = ptid; i < KB; i += 128 * NPG) {
            sw_s[i] = __ldg(args.w_scale0 + wrow + i);
            if (C::kTwoA) sw_s[KB + i] = __ldg(ws1 + i);
          }
        }
        if (!group_sync()) {
          ok = false;
          break;
        }
      }

      float acc0[C::kCols], acc1[C::kTwoA ? C::kCols : 1];
#pragma unroll
      for (int j = 0; j < C::kCols; ++j) {
        acc0[j] = 0.f;
        if (C::kTwoA) acc1[j] = 0.f;
      }
      const uint32_t tq = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
      for (int pg = 0; pg < NP; ++pg, ++pit) {
        const int pb = pit % C::kPBufs;
        if (!mbar_wait(&pfull[pb], (pit / C::kPBufs) & 1u, abort_flag, lim)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const float sw0 = FP8 && !C::kPreMul ? sw_s[pg] : 1.f;
        const float sw1 = (FP8 && C::kTwoA && !C::kPreMul) ? sw_s[KB + pg] : 0.f;
        const float* sa = sa_s + pg * BN + c_begin;
        const float* sb = sb_s + pg * BN + c_begin;
        // loads in batches of kBatch columns, one wait per batch, then the
        // arithmetic: tcgen05.wait::ld waits for all outstanding loads, so a
        // wait per 16-column chunk would pay the TMEM round trip once per
        // chunk; with three groups the registers allow batches of 16 only
#pragma unroll
        for (int b0 = 0; b0 < C::kCols; b0 += C::kBatch) {
          uint32_t g[C::kBatch], v[C::kTwoA ? C::kBatch : 1];
#pragma unroll
          for (int c = 0; c < C::kBatch / 16; ++c) {
            if (c_begin + b0 + c * 16 < un.nvalid) {
              tmem_ld16(tq + pb * C::kPCols + c_begin + b0 + c * 16,
                        *reinterpret_cast<uint32_t(*)[16]>(&g[c * 16]));
              if (C::kTwoA)
                tmem_ld16(tq + pb * C::kPCols + BN + c_begin + b0 + c * 16,
                          *reinterpret_cast<uint32_t(*)[16]>(&v[c * 16]));
            }
          }
          tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < C::kBatch / 16; ++c) {
            if (c_begin + b0 + c * 16 < un.nvalid) {
              if (FP8) {
                // acc += partial * (s_w * s_x[row]): four activation scales per
                // 16-byte load (all lanes read the same address), then pairs
                // of columns per packed multiply and multiply-add
#pragma unroll
                for (int jj = c * 16; jj < c * 16 + 16; jj += 4) {
                  const int j = b0 + jj;
                  const float4 s4 = *reinterpret_cast<const float4*>(sa + j);
                  float c00 = s4.x, c01 = s4.y, c02 = s4.z, c03 = s4.w;
                  if (!C::kPreMul) {
                    mul2(c00, c01, sw0, sw0, s4.x, s4.y);
                    mul2(c02, c03, sw0, sw0, s4.z, s4.w);
                  }
                  fma2(acc0[j], acc0[j + 1], __uint_as_float(g[jj]), __uint_as_float(g[jj + 1]),
                       c00, c01);
                  fma2(acc0[j + 2], acc0[j + 3], __uint_as_float(g[jj + 2]),
                       __uint_as_float(g[jj + 3]), c02, c03);
                  if (C::kTwoA) {
                    float c10, c11, c12, c13;
                    if (C::kPreMul) {
                      const float4 t4 = *reinterpret_cast<const float4*>(sb + j);
                      c10 = t4.x;
                      c11 = t4.y;
                      c12 = t4.z;
                      c13 = t4.w;
                    } else {
                      mul2(c10, c11, sw1, sw1, s4.x, s4.y);
                      mul2(c12, c13, sw1, sw1, s4.z, s4.w);
                    }
                    fma2(acc1[j], acc1[j + 1], __uint_as_float(v[jj]), __uint_as_float(v[jj + 1]),
                         c10, c11);
                    fma2(acc1[j + 2], acc1[j + 3], __uint_as_float(v[jj + 2]),
                         __uint_as_float(v[jj + 3]), c12, c13);
                  }
                }
              } else {
#pragma unroll
                for (int jj = c * 16; jj < c * 16 + 16; ++jj) acc0[b0 + jj] += __uint_as_float(g[jj]);
              }
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&pempty[pb]);
      }
      if (!ok) break;

      const int feat = un.mt * 128 + q * 32 + lane;
      if (GATED) {
        // h = silu(g) * u, then per-row e4m3 quantisation over this tile's 128 features
        uint8_t* hq = static_cast<uint8_t*>(args.out);
#pragma unroll
        for (int j = 0; j < C::kCols; ++j) {
          const float gv = acc0[j];
          acc0[j] = gv / (1.f + expf(-gv)) * acc1[j];
          if (c_begin + j < un.nvalid) {
            const uint32_t m = __reduce_max_sync(0xffffffffu, __float_as_uint(fabsf(acc0[j])));
            if (lane == 0) amax_s[q * BN + c_begin + j] = __uint_as_float(m);
          }
        }
        if (!group_sync()) {
          ok = false;
          break;
        }
#pragma unroll
        for (int j = 0; j < C::kCols; ++j) {
          const int col = c_begin + j;
          if (col < un.nvalid) {
            const float amax = fmaxf(fmaxf(amax_s[col], amax_s[BN + col]),
                                     fmaxf(amax_s[2 * BN + col], amax_s[3 * BN + col]));
            const float sh = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
            const size_t row = static_cast<size_t>(un.row0 + col);
            float2 pair;
            pair.x = __fdiv_rn(acc0[j], sh);
            pair.y = 0.f;
            const __nv_fp8x2_storage_t b = __nv_cvt_float2_to_fp8x2(pair, __NV_SATFINITE, __NV_E4M3);
            hq[row * args.ld + feat] = static_cast<uint8_t>(b & 0xFF);
            if (q == 0 && lane == 0) args.out_scale[row * args.m_tiles + un.mt] = sh;
          }
        }
      } else {
        // expert outputs (down) in BF16; router logit partials in fp32
        auto put = [&](size_t i, float v) {
          if (args.out_bf16) static_cast<__nv_bfloat16*>(args.out)[i] = __float2bfloat16_rn(v);
          else static_cast<float*>(args.out)[un.split * args.split_stride + i] = v;
        };
        const int f0 = DUAL ? un.mt * 256 + q * 32 + lane : feat;
        if (f0 < args.m_valid) {
#pragma unroll
          for (int j = 0; j < C::kCols; ++j)
            if (c_begin + j < un.nvalid)
              put(static_cast<size_t>(un.row0 + c_begin + j) * args.ld + f0, acc0[j]);
        }
        if (DUAL && f0 + 128 < args.m_valid) {
#pragma unroll
          for (int j = 0; j < C::kCols; ++j)
            if (c_begin + j < un.nvalid)
              put(static_cast<size_t>(un.row0 + c_begin + j) * args.ld + f0 + 128, acc1[j]);
        }
      }
    }
    if (!ok && lane == 0) {
      *abort_flag = 1;
      atomicOr(args.status, MOE_DEVICE_WAIT_TIMEOUT);
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (*abort_flag && warp == 0 && lane == 0) {
    for (uint32_t j = *consumed; j < *issued; ++j)
      mbar_wait(&full[j % S], (j / S) & 1u, nullptr);
  }
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, C::kTmemCols);
}

template <int BN, bool GATED, bool FP8, int NPG, bool DUAL = false>
static cudaError_t launch_one(moe_handle* h, const CUtensorMap& a0, const CUtensorMap& a1,
                              const CUtensorMap& b, GemmArgs args, cudaStream_t s) {
  using C = PromCfg<BN, GATED, FP8, NPG, DUAL>;
  auto kern = grouped_gemm_promoted_kernel<BN, GATED, FP8, NPG, DUAL>;
  static bool configured[64] = {};
  if (h->device < 64 && !configured[h->device]) {
    cudaError_t e = cudaFuncSetAttribute(kern,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kPromSmemBudget + 1024);
    if (e != cudaSuccess) return e;
    configured[h->device] = true;
  }
  args.stages = C::stages(args.k_blocks);
  if (args.stages < 2) return cudaErrorInvalidValue;
  const int smem = C::smem(args.k_blocks);
  kern<<<h->num_sms, C::kThreads, smem, s>>>(
      a0, a1, b, args);
  h->launches++;
  const cudaError_t e = cudaGetLastError();
  if (e == cudaErrorLaunchOutOfResources) {
    cudaFuncAttributes fa{};
    cudaFuncGetAttributes(&fa, kern);
    char buf[256];
    snprintf(buf, sizeof buf,
             "promoted GEMM BN=%d: %d threads x %d registers, %zu B local, max threads %d, "
             "%d B dynamic smem",
             BN, C::kThreads, fa.numRegs, fa.localSizeBytes, fa.maxThreadsPerBlock, smem);
    h->last_error = buf;
  }
  return e;
}

cudaError_t launch_gemm_fp8(moe_handle* h, bool gated, const GemmPlan& p, cudaStream_t s) {
  const Dims& dm = h->dims;
  if (p.k_blocks > kFp8MaxKBlocks) return cudaErrorInvalidValue;
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
    a.out_scale = h->ws.hs;
    a.w_scale0 = h->w.gate_s;
    a.w_scale1 = h->w.up_s;
    // short tiles gather the token rows (and scales) of the once-quantised
    // x; taller ones read rows quantised into expert order by the dispatch
    a.act_scale = h->ws.xs;
    a.row_token = p.gather ? h->ws.row_token : nullptr;
    const CUtensorMap& b = p.gather ? h->tm_xg : h->tm_xp[bi];
    const CUtensorMap &g = h->tm_gate, &u = h->tm_up;
    switch (p.bn) {
      case 16: return launch_one<16, true, true, 1>(h, g, u, b, a, s);
      case 32: return launch_one<32, true, true, 1>(h, g, u, b, a, s);
      case 64: return launch_one<64, true, true, SMOE_FP8_GU64_NPG>(h, g, u, b, a, s);
      case 96: return launch_one<96, true, true, 3>(h, g, u, b, a, s);
      default: return cudaErrorInvalidValue;
    }
  }
  a.out = h->ws.out;
  a.out_bf16 = 1;
  a.ld = dm.d;
  a.w_scale0 = h->w.down_s;
  a.w_scale1 = h->w.down_s;
  a.act_scale = h->ws.hs;
  const CUtensorMap& b = h->tm_h[bi];
  const CUtensorMap& w = h->tm_down;
  if (p.na == 2) {
    switch (p.bn) {
      case 16: return launch_one<16, false, true, 1, true>(h, w, w, b, a, s);
      case 32: return launch_one<32, false, true, 1, true>(h, w, w, b, a, s);
      case 64: return launch_one<64, false, true, 2, true>(h, w, w, b, a, s);
      default: return cudaErrorInvalidValue;
    }
  }
  switch (p.bn) {
    case 16: return launch_one<16, false, true, 1>(h, w, w, b, a, s);
    case 32: return launch_one<32, false, true, 1>(h, w, w, b, a, s);
    case 64: return launch_one<64, false, true, 1>(h, w, w, b, a, s);
    case 128: return launch_one<128, false, true, 2>(h, w, w, b, a, s);
    case 192: return launch_one<192, false, true, 3>(h, w, w, b, a, s);
    default: return cudaErrorInvalidValue;
  }
}

// Router logits on the tensor cores: logits[t, e] = x_t . W_g[e] with the fp32
// router weight held as three BF16 parts W = hi + mid + lo (exact: 3 x 8
// significand bits cover fp32's 24), concatenated along K. x (BF16) times
// each part is an exact product; partial sums over 128 K are promoted into
// fp32 registers (see the file comment). One group of T rows; B's K index
// wraps onto x's d columns. Each part is its own K slice (kTensorRouterSplits
// partial logits, added by the top-k kernel), which also triples the units so
// that the grid runs close to whole waves.
cudaError_t launch_router_gemm(moe_handle* h, const void* x, int T, cudaStream_t s) {
  const Dims& dm = h->dims;
  constexpr int BN = 256;  // tokens per tile: a 64-K stage holds 512 cycles of MMA work
  CUtensorMap tmx;
  {
    uint64_t dims[2] = {static_cast<uint64_t>(dm.d), static_cast<uint64_t>(T)};
    uint64_t str[1] = {static_cast<uint64_t>(dm.d) * 2};
    uint32_t box[2] = {64, BN};
    std::string err;
    if (!make_tmap(&tmx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(x), dims, str, box,
                   &err))
      return cudaErrorInvalidValue;
  }
  GemmArgs a{};
  a.offsets = nullptr;
  a.unit_base = nullptr;
  a.G = 1;
  a.single_rows = T;
  a.m_tiles = (dm.E + 127) / 128;
  a.k_blocks = 3 * dm.d / 64;
  a.ksplit = kTensorRouterSplits;
  a.split_stride = static_cast<size_t>(T) * dm.E;
  // the high BF16 part is promoted every 128 K (its fp32 partial sums carry
  // the logit's magnitude); the middle and low parts are 2^-8 and 2^-16 of
  // it, so the tensor core's own accumulation over their whole slice adds
  // error far below the 1e-5 band: one promotion per slice
  a.kpp = 2;
  a.kpp_rest = a.k_blocks / kTensorRouterSplits;
  a.bn = BN;
  a.b_k = dm.d;
  a.m_valid = dm.E;
  a.out = h->ws.logits_part;
  a.ld = dm.E;
  a.status = h->ws.status;
  return launch_one<BN, false, false, 4>(h, h->tm_router, h->tm_router, tmx, a, s);
}

}  // namespace smoe
