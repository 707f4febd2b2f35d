// ffn_fused.cu - the expert FFN of fine-grained experts in one kernel:
// gate/up GEMM, SwiGLU and down GEMM, with H kept on chip.
//
// For each expert-grouped row r of expert e (token t):
//   H_r      = silu(x_t W_g[e]) * (x_t W_u[e])            (bf16, never stored)
//   Y_perm_r = H_r W_d[e]                                  (bf16)
// (SwiGLU experts: "Revisiting MoE and Dense Speed-Accuracy Comparisons",
// 2.1 Architecture.)  The arithmetic of every output is the one of the
// separate grouped GEMMs (same MMA shapes along K, same bf16 rounding of H),
// so Y_perm is identical to that path.
//
// When f is small the whole H tile of 128 rows fits in tensor memory and
// shared memory, so H never travels to global memory and the three stages
// of a tile overlap inside one persistent CTA per SM:
//   warp 0 (+ warps 15-17 in gather mode)  producer: the 128 x 64 A blocks
//           (rows of x through the permutation, by cp.async in gather mode,
//           else TMA tiles of x_perm) with the matching W_g/W_u block into a
//           ring
//   warp 1  MMA1: acc1 = A W_gu^T (M 128, N 2f) into one of two TMEM
//           accumulators (allocates TMEM)
//   warp 2  MMA2: acc2 = H W_d^T (M 128, N d) from the H tile in shared
//           memory; it also loads each tile's W_d [d x f] by TMA into one
//           buffer, the next tile's as soon as the down GEMM has read it.
//           Separate issuing threads, so neither GEMM's waits hold up the
//           other (one thread issuing both measured a bubble: each down GEMM
//           waited for the next tile's rows)
//   warps 3-6   SwiGLU: acc1 -> bf16 H rows written in the 128-byte-swizzled
//               K-major layout the down GEMM reads (double-buffered)
//   warps 7-14  down epilogue: acc2 -> bf16 Y_perm rows (staged per warp,
//               stored in whole 64-byte row segments)
// The gate-weighted combine stays a separate kernel: folding it in (per-token
// arrival counters, the last arrival summing the k rows) measured slower on
// B200 -- its fences and reads sat on the epilogue's critical path while the
// Y_perm writes already bound the tile rate.
// Every wait is bounded; a wait that gives up records
// MOE_ERR_DEVICE_TIMEOUT, stops the other roles, drains in-flight copies and
// MMAs, and frees TMEM.
#include <cudaTypedefs.h>

#include "kernels.cuh"

namespace moe {

namespace {

constexpr int BM = 128, BK = 64;
constexpr int kGatherWarps = 4;
constexpr int kEpi1Warps = 4;
constexpr int kEpi2Warps = 8;
constexpr int kMma1Warp = 1, kMma2Warp = 2;
constexpr int kEpi1First = 3, kEpi2First = 7, kGatherFirst = 15;

template <bool GATHER>
constexpr int ffn_threads() { return 32 * (kGatherFirst + (GATHER ? kGatherWarps - 1 : 0)); }

template <int F, int D>
struct Cfg {
  static constexpr int NA1 = (4 * F + D <= 512) ? 2 : 1;  // gate/up accumulators
  static constexpr uint32_t A2_COL = NA1 * 2 * F;         // TMEM column of acc2
  static constexpr uint32_t TMEM_COLS = 512;
  static_assert(A2_COL + D <= TMEM_COLS, "accumulators fit in tensor memory");
  static constexpr uint32_t A_BYTES = BM * BK * 2;
  static constexpr uint32_t B1_BYTES = 2 * F * BK * 2;
  static constexpr uint32_t STAGE = A_BYTES + B1_BYTES;
  static constexpr uint32_t WD_KBLK = D * BK * 2;  // one 64-wide K block of W_d
  static constexpr uint32_t WD_BYTES = WD_KBLK * (F / BK);
  static constexpr uint32_t H_KBLK = BM * BK * 2;
  static constexpr uint32_t H_BYTES = H_KBLK * (F / BK);
  static constexpr uint32_t STG_ROW = 64 + 16;  // per-warp staging row: 32 bf16 + pad
  static constexpr uint32_t STG_WARP = 32 * STG_ROW;
  static constexpr uint32_t STG_BYTES = kEpi2Warps * STG_WARP;
  static constexpr uint32_t BUDGET = 222u * 1024u;  // of the 227 KB a CTA may use
  static constexpr int NHB = (2 * H_BYTES + WD_BYTES + 3 * STAGE + STG_BYTES <= BUDGET) ? 2 : 1;
  static constexpr int STAGES_RAW = (int)((BUDGET - WD_BYTES - NHB * H_BYTES - STG_BYTES) / STAGE);
  static constexpr int STAGES = STAGES_RAW > 6 ? 6 : (STAGES_RAW < 2 ? 2 : STAGES_RAW);
  static constexpr size_t SMEM = (size_t)STAGES * STAGE + WD_BYTES + NHB * H_BYTES + STG_BYTES + 1024;
  static constexpr int KB1 = D / BK;
  static constexpr int KB2 = F / BK;
  static constexpr uint32_t IDESC1 = idesc_bf16_f32(BM, 2 * F);
  static constexpr uint32_t IDESC2 = idesc_bf16_f32(BM, D);
};

struct Params {
  const int32_t* offsets;  // [G + 1] expert row offsets
  const void* A;           // gather: x [src_rows, D]; else x_perm [rows, D]
  const int32_t* gather;   // gather: row_token (A row r is x row gather[r])
  int64_t src_rows, rows;
  int G;
  __nv_bfloat16* y_perm;  // [rows, D]
  Control* ctl;
};

struct TileInfo {
  int g, row0, rows;
};

__device__ __forceinline__ TileInfo decode(int mt, const int* tile_off, const int* s_off, int G) {
  TileInfo ti;
  int lo = 1, hi = G;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (tile_off[mid] > mt) hi = mid; else lo = mid + 1;
  }
  ti.g = lo - 1;
  ti.row0 = s_off[ti.g] + (mt - tile_off[ti.g]) * BM;
  ti.rows = min(BM, s_off[ti.g + 1] - ti.row0);
  return ti;
}

__device__ __forceinline__ float silu_mul(float g, float u) {
  return __fdividef(g, 1.f + __expf(-g)) * u;
}

template <int F, int D, bool GATHER>
__global__ void __launch_bounds__(ffn_threads<GATHER>(), 1)
    ffn_fused_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB1,
                     const __grid_constant__ CUtensorMap tmB2, const __grid_constant__ Params p) {
  using C = Cfg<F, D>;
  constexpr int STAGES = C::STAGES, NA1 = C::NA1, NHB = C::NHB;
  constexpr int NT = ffn_threads<GATHER>();

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sRing = smem;                                // STAGES x (A | B1)
  uint8_t* sWd = sRing + STAGES * C::STAGE;             // W_d tile
  uint8_t* sH = sWd + C::WD_BYTES;                      // NHB x H tile
  uint8_t* sStg = sH + NHB * C::H_BYTES;                // per-warp staging (down epilogue)

  __shared__ __align__(8) uint64_t full[STAGES], empty[STAGES], wfull, wempty;
  __shared__ __align__(8) uint64_t a1full[NA1], a1empty[NA1], hfull[NHB], hempty[NHB];
  __shared__ __align__(8) uint64_t a2full, a2empty, done;
  __shared__ uint32_t tmem_base_s;
  __shared__ int tile_off[257];
  __shared__ int s_off[257];
  __shared__ volatile int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.G;

  // setup that reads nothing the previous kernel writes runs before the
  // dependency wait: barriers, tensor memory, descriptor prefetch
  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], GATHER ? 32 * kGatherWarps + 1 : 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(&wfull, 1);
    mbar_init(&wempty, 1);
    for (int b = 0; b < NA1; ++b) {
      mbar_init(&a1full[b], 1);
      mbar_init(&a1empty[b], kEpi1Warps);
    }
    for (int b = 0; b < NHB; ++b) {
      mbar_init(&hfull[b], kEpi1Warps);
      mbar_init(&hempty[b], 1);
    }
    mbar_init(&a2full, 1);
    mbar_init(&a2empty, kEpi2Warps);
    mbar_init(&done, 2);  // one commit per MMA-issuing thread
    fence_barrier_init();
    if (!GATHER) tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB1);
    tma_prefetch_desc(&tmB2);
  } else if (warp == kMma1Warp) {
    tmem_alloc(&tmem_base_s, C::TMEM_COLS);
    tmem_relinquish();
  }
  __syncwarp();
  pdl_wait();
  for (int g = threadIdx.x; g <= G; g += NT)
    s_off[g] = min(max(__ldg(p.offsets + g), 0), (int)p.rows);
  __syncthreads();
  if (warp == 0) {
    int carry = 0;
    for (int g0 = 0; g0 < G; g0 += 32) {
      const int g = g0 + lane;
      const int v = g < G ? (max(s_off[g + 1] - s_off[g], 0) + BM - 1) / BM : 0;
      int incl = v;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
      }
      if (g < G) tile_off[g] = carry + incl - v;
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) tile_off[G] = carry;
  }
  tc_fence_before();
  __syncwarp();  // role branches diverged single lanes: reconverge before the CTA barrier
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_base_s;
  const int total = tile_off[G];

  const bool gather_warp = GATHER && (warp == 0 || warp >= kGatherFirst);
  if (warp == 0 || gather_warp) {
    // ------------------------------------------------------------ producer
    constexpr int RPW = BM / kGatherWarps;
    const int gw = warp == 0 ? 0 : warp - (kGatherFirst - 1);
    const int ch = lane & 7, rsub = lane >> 3;
    uint32_t it = 0;
    bool ok = true;
    int32_t src[RPW / 4], nxt[RPW / 4];
    auto load_src = [&](int tile, int32_t (&dst)[RPW / 4]) {
      const TileInfo t2 = decode(tile, tile_off, s_off, G);
#pragma unroll
      for (int i = 0; i < RPW / 4; ++i) {
        const int64_t r = (int64_t)t2.row0 + gw * RPW + 4 * i + rsub;
        dst[i] = r < p.rows ? __ldg(p.gather + r) : 0;
      }
    };
    if (GATHER && blockIdx.x < total) load_src(blockIdx.x, nxt);
    for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
      const TileInfo ti = decode(tile, tile_off, s_off, G);
      if constexpr (GATHER) {
#pragma unroll
        for (int i = 0; i < RPW / 4; ++i) src[i] = (nxt[i] >= 0 && nxt[i] < p.src_rows) ? nxt[i] : 0;
        if (tile + (int)gridDim.x < total) load_src(tile + gridDim.x, nxt);
      }
      for (int kb = 0; kb < C::KB1; ++kb, ++it) {
        const uint32_t s = it % STAGES, ph = (it / STAGES) & 1;
        uint8_t* sA = sRing + s * C::STAGE;
        int good = 1;
        if (lane == 0) {
          good = mbar_wait_bounded(&empty[s], ph ^ 1, &abort_flag);
          if (good && gw == 0) {
            mbar_arrive_expect_tx(&full[s], GATHER ? C::B1_BYTES : C::STAGE);
            if (!GATHER) tma_load_2d(sA, &tmA, &full[s], kb * BK, ti.row0);
            tma_load_2d(sA + C::A_BYTES, &tmB1, &full[s], kb * BK, ti.g * 2 * F);
          }
        }
        good = __shfl_sync(0xffffffffu, good, 0);
        if (!good) {
          ok = false;
          break;
        }
        if constexpr (GATHER) {
          const __nv_bfloat16* xa = static_cast<const __nv_bfloat16*>(p.A) + kb * BK + ch * 8;
          const uint32_t sa = smem_u32(sA);
#pragma unroll
          for (int i = 0; i < RPW / 4; ++i) {
            const int r = gw * RPW + 4 * i + rsub;
            cp_async_16(sa + r * 128 + ((ch ^ (r & 7)) << 4), xa + (int64_t)src[i] * D);
          }
          cp_async_arrive_noinc(&full[s]);
        }
      }
    }
    if (lane == 0 && !ok) {
      abort_flag = 1;
      record_error(p.ctl, MOE_ERR_DEVICE_TIMEOUT, 0x600u);
    }
    if constexpr (GATHER) cp_async_wait_all();
    // drain: issued copies land before the CTA may exit
    if (gw == 0 && lane == 0) {
      const uint32_t first = it > (uint32_t)STAGES ? it - STAGES : 0;
      for (uint32_t q = first; q < it; ++q) mbar_wait_bounded(&full[q % STAGES], (q / STAGES) & 1, nullptr);
    }
  } else if (warp == kMma1Warp) {
    // ---------------------------------------------------------------- MMA1
    if (lane == 0) {
      uint32_t it = 0, i = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x, ++i) {
        // acc1[i % NA1] = A W_gu^T over D
        const uint32_t ab = i % NA1, aph = (i / NA1) & 1;
        if (!mbar_wait_bounded(&a1empty[ab], aph ^ 1, &abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d1 = tmem_base + ab * 2 * F;
        for (int kb = 0; kb < C::KB1; ++kb, ++it) {
          const uint32_t s = it % STAGES, ph = (it / STAGES) & 1;
          if (!mbar_wait_bounded(&full[s], ph, &abort_flag)) {
            ok = false;
            break;
          }
          if constexpr (GATHER) fence_proxy_async_shared();  // cp.async rows -> tensor core
          tc_fence_after();
          const uint32_t a0 = smem_u32(sRing + s * C::STAGE);
          const uint32_t b0 = a0 + C::A_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            tc_mma_f16(d1, smem_desc_k128(a0 + kk * 32), smem_desc_k128(b0 + kk * 32), C::IDESC1,
                       (kb | kk) != 0);
          tc_commit(&empty[s]);
        }
        if (!ok) break;
        tc_commit(&a1full[ab]);
      }
      if (!ok) {
        abort_flag = 1;
        record_error(p.ctl, MOE_ERR_DEVICE_TIMEOUT, 0x700u);
      }
      // this thread's MMAs complete before TMEM is released
      tc_commit(&done);
      mbar_wait_bounded(&done, 0, nullptr);
    }
  } else if (warp == kMma2Warp) {
    // ---------------------------------------------------------------- MMA2
    // This warp also loads each tile's W_d [D x F] (F / 64 blocks of D rows
    // x 64) into the single W_d buffer: the next tile's as soon as this
    // tile's down GEMM has completed, while the SwiGLU of the next tile is
    // still running.
    if (lane == 0) {
      uint32_t j = 0;
      bool ok = true;
      auto load_wd = [&](int tile) {
        const TileInfo ti = decode(tile, tile_off, s_off, G);
        mbar_arrive_expect_tx(&wfull, C::WD_BYTES);
        for (int kb = 0; kb < C::KB2; ++kb)
          tma_load_2d(sWd + kb * C::WD_KBLK, &tmB2, &wfull, kb * BK, ti.g * D);
      };
      if (blockIdx.x < total) load_wd(blockIdx.x);
      for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++j) {
        // acc2 = H W_d^T over F
        const uint32_t hb = j % NHB;
        if (!mbar_wait_bounded(&hfull[hb], (j / NHB) & 1, &abort_flag) ||
            !mbar_wait_bounded(&wfull, j & 1, &abort_flag) ||
            !mbar_wait_bounded(&a2empty, (j & 1) ^ 1, &abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d2 = tmem_base + C::A2_COL;
#pragma unroll
        for (int kb = 0; kb < C::KB2; ++kb) {
          const uint32_t h0 = smem_u32(sH + hb * C::H_BYTES + kb * C::H_KBLK);
          const uint32_t w0 = smem_u32(sWd + kb * C::WD_KBLK);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            tc_mma_f16(d2, smem_desc_k128(h0 + kk * 32), smem_desc_k128(w0 + kk * 32), C::IDESC2,
                       (kb | kk) != 0);
        }
        tc_commit(&hempty[hb]);
        tc_commit(&wempty);
        tc_commit(&a2full);
        if (tile + (int)gridDim.x < total) {
          // W_d of the next tile once this down GEMM has read the buffer
          if (!mbar_wait_bounded(&wempty, j & 1, &abort_flag)) {
            ok = false;
            break;
          }
          load_wd(tile + gridDim.x);
        }
      }
      if (!ok) {
        abort_flag = 1;
        record_error(p.ctl, MOE_ERR_DEVICE_TIMEOUT, 0x780u);
      }
      // every MMA of this CTA is issued: let the next kernel's CTAs be
      // scheduled (they still wait for this grid to complete)
      pdl_trigger();
      // a W_d load issued for a tile that was not reached (error path) lands
      // before the CTA may exit
      if (!ok) mbar_wait_bounded(&wfull, j & 1, nullptr);
      tc_commit(&done);
      mbar_wait_bounded(&done, 0, nullptr);
    }
  } else if (warp < kEpi2First) {
    // ------------------------------------------------------------- SwiGLU
    const int q = warp & 3;
    const int rr = q * 32 + lane;
    uint32_t i = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++i) {
      const uint32_t ab = i % NA1, hb = i % NHB;
      if (!mbar_wait_bounded(&a1full[ab], (i / NA1) & 1, &abort_flag) ||
          !mbar_wait_bounded(&hempty[hb], ((i / NHB) & 1) ^ 1, &abort_flag)) {
        abort_flag = 1;
        record_error(p.ctl, MOE_ERR_DEVICE_TIMEOUT, 0x800u);
        break;
      }
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + ab * 2 * F;
      uint8_t* hrow = sH + hb * C::H_BYTES + rr * 128;
#pragma unroll 1
      for (int c = 0; c < F; c += 16) {
        uint32_t g0[16], u0[16];
        tmem_ld16(taddr + c, g0);
        tmem_ld16(taddr + F + c, u0);
        tmem_ld_wait();
        uint32_t pk[8];
#pragma unroll
        for (int v = 0; v < 8; ++v)
          pk[v] = pack_bf16x2(silu_mul(__uint_as_float(g0[2 * v]), __uint_as_float(u0[2 * v])),
                              silu_mul(__uint_as_float(g0[2 * v + 1]), __uint_as_float(u0[2 * v + 1])));
        // columns c .. c+15 = chunks (c % 64) / 8 and +1 of K block c / 64;
        // chunk x of row r is stored at x ^ (r % 8) (128-byte swizzle)
        uint8_t* kbase = hrow + (c / BK) * C::H_KBLK;
        const int x0 = (c % BK) / 8;
#pragma unroll
        for (int v = 0; v < 2; ++v)
          *reinterpret_cast<uint4*>(kbase + (((x0 + v) ^ (rr & 7)) << 4)) =
              make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
      }
      tc_fence_before();
      fence_proxy_async_shared();  // H rows -> tensor core
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&a1empty[ab]);
        mbar_arrive(&hfull[hb]);
      }
    }
  } else if (warp < kEpi2First + kEpi2Warps) {
    // -------------------------------------------------------- down epilogue
    const int q = warp & 3;
    const int h = (warp - kEpi2First) >> 2;
    const int w8 = warp - kEpi2First;
    constexpr int HALF = D / 2;
    uint8_t* stg = sStg + w8 * C::STG_WARP;
    uint32_t i = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++i) {
      const TileInfo ti = decode(tile, tile_off, s_off, G);
      if (!mbar_wait_bounded(&a2full, i & 1, &abort_flag)) {
        abort_flag = 1;
        record_error(p.ctl, MOE_ERR_DEVICE_TIMEOUT, 0x900u);
        break;
      }
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + C::A2_COL + h * HALF;
      // rounds of 32 columns; the next round's TMEM loads are in flight while
      // this round is staged and stored, and the accumulator is released as
      // soon as its last columns are in registers
      uint32_t r0[16], r1[16];
      tmem_ld16(taddr, r0);
      tmem_ld16(taddr + 16, r1);
      tmem_ld_wait();
#pragma unroll 1
      for (int c = 0; c < HALF; c += 32) {
        uint32_t pk[16];
#pragma unroll
        for (int v = 0; v < 8; ++v) {
          pk[v] = pack_bf16x2(__uint_as_float(r0[2 * v]), __uint_as_float(r0[2 * v + 1]));
          pk[8 + v] = pack_bf16x2(__uint_as_float(r1[2 * v]), __uint_as_float(r1[2 * v + 1]));
        }
        if (c + 32 < HALF) {
          tmem_ld16(taddr + c + 32, r0);
          tmem_ld16(taddr + c + 48, r1);
        } else {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&a2empty);
        }
        // this lane's 32 columns -> its staging row (64 bytes)
        uint4* srow = reinterpret_cast<uint4*>(stg + lane * C::STG_ROW);
#pragma unroll
        for (int v = 0; v < 4; ++v) srow[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
        __syncwarp();
        // copy-out: 8 rows x 64 bytes per instruction (4 lanes a row)
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const int r = 8 * m + (lane >> 2), cc = lane & 3;
          const uint4 v = *reinterpret_cast<const uint4*>(stg + r * C::STG_ROW + cc * 16);
          if (q * 32 + r < ti.rows)
            *reinterpret_cast<uint4*>(p.y_perm + ((int64_t)ti.row0 + q * 32 + r) * D + h * HALF + c + cc * 8) = v;
        }
        __syncwarp();
        if (c + 32 < HALF) tmem_ld_wait();
      }
    }
  }

  tc_fence_before();
  __syncwarp();  // role branches diverged single lanes: reconverge before the CTA barrier
  __syncthreads();
  if (warp == kMma1Warp) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

template <int F, int D, bool GATHER>
cudaError_t run(const FfnArgs& a, cudaStream_t s) {
  using C = Cfg<F, D>;
  cudaError_t e = set_smem_limit((const void*)ffn_fused_kernel<F, D, GATHER>, C::SMEM);
  if (e != cudaSuccess) return e;
  CUtensorMap mA, mB1, mB2;
  // gather mode reads A with cp.async; its tensor map is built but unused
  if (!make_kmajor_map(&mA, a.A, GATHER ? a.src_rows : a.rows, D, BM)) return cudaErrorInvalidValue;
  if (!make_kmajor_map(&mB1, a.wgu, (int64_t)a.G * 2 * F, D, 2 * F)) return cudaErrorInvalidValue;
  if (!make_kmajor_map(&mB2, a.wdT, (int64_t)a.G * D, F, D)) return cudaErrorInvalidValue;
  Params p;
  p.offsets = a.offsets;
  p.A = a.A;
  p.gather = a.gather;
  p.src_rows = a.src_rows;
  p.rows = a.rows;
  p.G = a.G;
  p.y_perm = static_cast<__nv_bfloat16*>(a.y_perm);
  p.ctl = a.ctl;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t tiles_max = (a.rows + BM - 1) / BM + a.G;
  const int grid = (int)std::min<int64_t>(tiles_max, (int64_t)sms);
  return launch_pdl(ffn_fused_kernel<F, D, GATHER>, dim3(grid), dim3(ffn_threads<GATHER>()),
                    C::SMEM, s, mA, mB1, mB2, p);
}

}  // namespace

bool ffn_fused_supported(int d, int f) {
  return (f == 64 || f == 128) && (d == 128 || d == 256);
}

cudaError_t launch_ffn_fused(const FfnArgs& a, cudaStream_t s) {
  if (a.rows == 0) return cudaSuccess;
  if (!ffn_fused_supported(a.d, a.f)) return cudaErrorInvalidValue;
  const bool g = a.gather != nullptr;
#define MOE_FFN_CASE(F, D) \
  if (a.f == F && a.d == D) return g ? run<F, D, true>(a, s) : run<F, D, false>(a, s);
  MOE_FFN_CASE(64, 256)
  MOE_FFN_CASE(64, 128)
  MOE_FFN_CASE(128, 256)
  MOE_FFN_CASE(128, 128)
#undef MOE_FFN_CASE
  return cudaErrorInvalidValue;
}

}  // namespace moe
