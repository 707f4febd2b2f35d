// gemm_tc.cu - grouped GEMM on the fifth-generation tensor cores (tcgen05).
//
// The only dense contraction of the layer.  For each group g (an expert)
// and each row r in [offsets[g], offsets[g+1]):
//   acc[r, n] = sum_k A[r, k] * B[g*n_per_group + n, k]
// with one of two epilogues:
//   kEpiSwiGLU  B holds, per block of BN/2 output columns, the gate rows then
//               the up rows of W_g / W_u; out = silu(acc_gate) * acc_up in
//               bf16 (SwiGLU: "Revisiting MoE and Dense Speed-Accuracy
//               Comparisons", 2.1 Architecture)
//   kEpiBF16    out = acc in bf16 (the down projection)
//
// Design (persistent: one CTA per SM, two for short K loops; 10 warps, 13
// in gather mode):
//   warp 0      TMA producer: 128 x 64 A tiles and BN x 64 B tiles, 128-byte
//               swizzle, into a STAGES-deep shared-memory ring (full/empty
//               mbarriers).  Gather mode: the A rows are rows of x picked by
//               the permutation, copied with cp.async into the same swizzled
//               layout by warp 0 and warps 10-12, 32 rows each
//   warp 1      allocates tensor memory (two BN-column fp32 accumulators) and
//               one lane issues tcgen05.mma (M=128, N=BN, K=16) from shared-
//               memory descriptors; tcgen05.commit frees smem stages and
//               hands finished accumulators to the epilogue
//   warps 2-9   epilogue, two warps per TMEM lane quadrant (each reads half
//               of its 32 rows' columns): tcgen05.ld, activation, bf16 rows
//               to global memory -- straight from registers, or (short K
//               loops) staged in shared memory and copied out by whole rows
//               per warp instruction;
//               predicated on the group's last row so a tile never writes
//               rows of the next expert
// The tile list is (group, 128-row tile, N tile), N fastest, walked with a
// static stride of gridDim.x.  Group row counts come from device memory (no
// host synchronisation); every CTA rebuilds the tile prefix in shared memory.
// Every wait is bounded: a wait that gives up records MOE_ERR_DEVICE_TIMEOUT,
// stops the other roles, drains in-flight copies and MMAs, and frees TMEM.
#include <cudaTypedefs.h>

#include <algorithm>

#include "kernels.cuh"

namespace moe {

namespace {

constexpr int BM = 128, BK = 64;
constexpr int kEpiWarps = 8;  // two per TMEM lane quadrant
// gather mode: the A rows of a stage are copied by this many warps (warp 0
// and the warps after the epilogue), 32 rows each
constexpr int kGatherWarps = 4;
// producer + MMA + epilogue (+ the extra gather warps)
template <bool GATHER>
constexpr int threads_for() { return 64 + 32 * kEpiWarps + (GATHER ? 32 * (kGatherWarps - 1) : 0); }

struct Params {
  const int32_t* offsets;  // NULL: a single group of `rows` rows
  const void* A;           // gather mode: the source matrix [src_rows, K]
  const int32_t* gather;   // gather mode: A row r is source row gather[r]
  int64_t src_rows;        // gather mode: rows of the source matrix
  int64_t rows;
  int G, K, n_per_group, n_out;
  void* out;
  int64_t ld_out;
  // 1: `out` and the row pitch are 32-byte aligned, so the unstaged
  // epilogue writes each row's 64-byte column group as two 32-byte stores
  int out_v8;
  Control* ctl;
};

template <int BN>
constexpr uint32_t tmem_cols_for() {
  return (2 * BN <= 32) ? 32 : (2 * BN <= 64) ? 64 : (2 * BN <= 128) ? 128 : (2 * BN <= 256) ? 256 : 512;
}

// output columns of one tile, and the padded bytes of one staged output row
template <int BN, int EPI>
constexpr int out_cols() { return EPI == kEpiSwiGLU ? BN / 2 : BN; }
template <int BN, int EPI>
constexpr uint32_t staged_row_bytes() { return out_cols<BN, EPI>() * 2 + 16; }

// Staged epilogue: each epilogue thread writes its output row into shared
// memory, then the quadrant's two warps copy the rows out with every store
// instruction covering whole contiguous row segments (one small bulk copy
// per row measured slower: the copy engine's issue rate bound the tile).
// Used when the K loop is short and the epilogue would otherwise dominate;
// it costs pipeline stages.
template <int BN, int EPI, bool STAGED>
constexpr uint32_t staging_bytes() { return STAGED ? 128u * staged_row_bytes<BN, EPI>() : 0u; }

// Short K loops also run two CTAs per SM (when both fit in tensor memory and
// the producer needs no per-tile register state), so one CTA's load latency
// overlaps the other's tiles.
template <int BN, bool STAGED, bool GATHER>
constexpr int ctas_per_sm() { return (STAGED && !GATHER && tmem_cols_for<BN>() <= 256) ? 2 : 1; }

template <int BN, int EPI, bool STAGED, bool GATHER>
constexpr int stages_for() {
  constexpr uint32_t stage = BM * BK * 2 + BN * BK * 2;
  constexpr uint32_t budget = (ctas_per_sm<BN, STAGED, GATHER>() == 2 ? 104u : 220u) * 1024u;
  constexpr uint32_t n = (budget - staging_bytes<BN, EPI, STAGED>()) / stage;
  return n > 8 ? 8 : (n < 2 ? 2 : (int)n);
}

template <int BN, int EPI, bool STAGED, bool GATHER>
constexpr size_t smem_bytes_for() {
  return (size_t)stages_for<BN, EPI, STAGED, GATHER>() * (BM * BK * 2 + BN * BK * 2) +
         staging_bytes<BN, EPI, STAGED>() + 1024;
}

struct TileInfo {
  int g, row0, rows, nt;
};

__device__ __forceinline__ TileInfo decode(int tile, int n_tiles, const int* tile_off,
                                           const int* s_off, int G) {
  TileInfo ti;
  const int mt = tile / n_tiles;
  ti.nt = tile - mt * n_tiles;
  // first i in [1, G] with tile_off[i] > mt  ->  group i - 1
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

template <int BN, int EPI, bool GATHER, bool STAGED>
__global__ void __launch_bounds__(threads_for<GATHER>(), (ctas_per_sm<BN, STAGED, GATHER>()))
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ Params p) {
  constexpr int STAGES = stages_for<BN, EPI, STAGED, GATHER>();
  constexpr uint32_t A_BYTES = BM * BK * 2;
  constexpr uint32_t B_BYTES = BN * BK * 2;
  constexpr uint32_t TMEM_COLS = tmem_cols_for<BN>();
  constexpr uint32_t IDESC = idesc_bf16_f32(BM, BN);
  constexpr uint32_t ACC_STRIDE = TMEM_COLS / 2;  // column distance of the two accumulators
  constexpr int NT = threads_for<GATHER>();

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * A_BYTES;
  uint8_t* sOut = smem + STAGES * (A_BYTES + B_BYTES);  // staged epilogue rows

  __shared__ __align__(8) uint64_t full[STAGES], empty[STAGES], tfull[2], tempty[2], done;
  __shared__ uint32_t tmem_base_s;
  __shared__ int tile_off[257];
  __shared__ int s_off[257];
  __shared__ volatile int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.G;

  // setup that reads nothing an earlier kernel writes runs before the
  // dependency wait: barriers, tensor memory, descriptor prefetch
  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int s = 0; s < STAGES; ++s) {
      // gather mode: the TMA arrival plus one cp.async arrival per lane of
      // every gather warp
      mbar_init(&full[s], GATHER ? 32 * kGatherWarps + 1 : 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], kEpiWarps);
    }
    mbar_init(&done, 1);
    fence_barrier_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  } else if (warp == 1) {
    tmem_alloc(&tmem_base_s, TMEM_COLS);
    tmem_relinquish();
  }
  __syncwarp();
  // everything below reads what earlier kernels wrote (offsets, operands)
  pdl_wait();
  // group offsets and the prefix of 128-row tiles per group; offsets clamped
  // to [0, rows]: a malformed offset array can never make the epilogue store
  // outside the output
  for (int g = threadIdx.x; g <= G; g += NT)
    s_off[g] = p.offsets ? min(max(__ldg(p.offsets + g), 0), (int)p.rows) : (g == 0 ? 0 : (int)p.rows);
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
  const int n_tiles = p.n_per_group / BN;
  const int total = tile_off[G] * n_tiles;
  const int kblocks = p.K / BK;

  const bool gather_warp = GATHER && (warp == 0 || warp >= 2 + kEpiWarps);
  if (warp == 0 || gather_warp) {
    if constexpr (GATHER) {
      // Permute fused into the operand load: the tile's 128 A rows are rows
      // gather[row0 .. row0+127] of the source (x).  Gather warp gw copies
      // rows 32*gw .. 32*gw+31 with 16-byte cp.async (lane l: chunk l%8 of
      // rows 32*gw + 4i + l/8), writing the 128-byte-swizzled layout a TMA
      // tile load would produce (chunk c of row r at c ^ (r % 8)); each
      // lane's copies arrive on the stage barrier when they land.  Warp 0
      // also loads B by TMA.  Rows past the end of the gather list read
      // source row 0; their results are never stored.
      constexpr int RPW = BM / kGatherWarps;  // rows per gather warp
      const int gw = warp == 0 ? 0 : warp - (1 + kEpiWarps);
      const int ch = lane & 7, rsub = lane >> 3;
      uint32_t it = 0;
      bool ok = true;
      // this warp's source rows of a tile; the next tile's are loaded while
      // the current one is copied, so their latency stays off the critical path
      auto load_src = [&](int tile, int32_t (&dst)[RPW / 4]) {
        const TileInfo t2 = decode(tile, n_tiles, tile_off, s_off, G);
#pragma unroll
        for (int i = 0; i < RPW / 4; ++i) {
          const int64_t r = (int64_t)t2.row0 + gw * RPW + 4 * i + rsub;
          dst[i] = r < p.rows ? __ldg(p.gather + r) : 0;
        }
      };
      int32_t src[RPW / 4], nxt[RPW / 4];
      if (blockIdx.x < total) load_src(blockIdx.x, nxt);
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        const TileInfo ti = decode(tile, n_tiles, tile_off, s_off, G);
        const int brow = ti.g * p.n_per_group + ti.nt * BN;
#pragma unroll
        for (int i = 0; i < RPW / 4; ++i) src[i] = (nxt[i] >= 0 && nxt[i] < p.src_rows) ? nxt[i] : 0;
        if (tile + (int)gridDim.x < total) load_src(tile + gridDim.x, nxt);
        for (int kb = 0; kb < kblocks; ++kb, ++it) {
          const uint32_t s = it % STAGES, ph = (it / STAGES) & 1;
          int good = 1;
          if (lane == 0) {
            good = mbar_wait_bounded(&empty[s], ph ^ 1, &abort_flag);
            if (good && gw == 0) {
              mbar_arrive_expect_tx(&full[s], B_BYTES);
              tma_load_2d(sB + s * B_BYTES, &tmB, &full[s], kb * BK, brow);
            }
          }
          good = __shfl_sync(0xffffffffu, good, 0);
          if (!good) {
            ok = false;
            break;
          }
          const __nv_bfloat16* xa = static_cast<const __nv_bfloat16*>(p.A) + kb * BK + ch * 8;
          const uint32_t sa = smem_u32(sA + s * A_BYTES);
#pragma unroll
          for (int i = 0; i < RPW / 4; ++i) {
            const int r = gw * RPW + 4 * i + rsub;
            cp_async_16(sa + r * 128 + ((ch ^ (r & 7)) << 4), xa + (int64_t)src[i] * p.K);
          }
          cp_async_arrive_noinc(&full[s]);
        }
      }
      if (lane == 0) {
        if (!ok) {
          abort_flag = 1;
          record_error(p.ctl, MOE_ERR_DEVICE_TIMEOUT, 0x100u);
        }
      }
      cp_async_wait_all();
      // drain: every issued stage (the B loads too) completes before the CTA
      // may exit
      if (gw == 0) {
        const uint32_t first = it > (uint32_t)STAGES ? it - STAGES : 0;
        for (uint32_t q = first; q < it; ++q)
          mbar_wait_bounded(&full[q % STAGES], (q / STAGES) & 1, nullptr);
      }
    } else if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        const TileInfo ti = decode(tile, n_tiles, tile_off, s_off, G);
        const int brow = ti.g * p.n_per_group + ti.nt * BN;
        for (int kb = 0; kb < kblocks; ++kb, ++it) {
          const uint32_t s = it % STAGES, ph = (it / STAGES) & 1;
          if (!mbar_wait_bounded(&empty[s], ph ^ 1, &abort_flag, true)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[s], A_BYTES + B_BYTES);
          tma_load_2d(sA + s * A_BYTES, &tmA, &full[s], kb * BK, ti.row0);
          tma_load_2d(sB + s * B_BYTES, &tmB, &full[s], kb * BK, brow);
        }
      }
      if (!ok) {
        abort_flag = 1;
        record_error(p.ctl, MOE_ERR_DEVICE_TIMEOUT, 0x100u);
      }
      // drain: every issued stage completes before the CTA may exit
      const uint32_t first = it > (uint32_t)STAGES ? it - STAGES : 0;
      for (uint32_t q = first; q < it; ++q)
        mbar_wait_bounded(&full[q % STAGES], (q / STAGES) & 1, nullptr);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      uint32_t it = 0, tc = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x, ++tc) {
        const uint32_t b = tc & 1, tph = (tc >> 1) & 1;
        if (!mbar_wait_bounded(&tempty[b], tph ^ 1, &abort_flag, true)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + b * ACC_STRIDE;
        for (int kb = 0; kb < kblocks; ++kb, ++it) {
          const uint32_t s = it % STAGES, ph = (it / STAGES) & 1;
          // the MMA thread and the TMA producer sleep in their waits
          // (mbar_try_wait_sleep); the gather warps spin, which measured faster
          if (!mbar_wait_bounded(&full[s], ph, &abort_flag, true)) {
            ok = false;
            break;
          }
          // cp.async wrote A through the generic proxy; the MMA reads it
          // through the async proxy
          if constexpr (GATHER) fence_proxy_async_shared();
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + s * A_BYTES);
          const uint32_t b0 = smem_u32(sB + s * B_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            tc_mma_f16(d_tmem, smem_desc_k128(a0 + kk * 32), smem_desc_k128(b0 + kk * 32), IDESC,
                       (kb | kk) != 0);
          tc_commit(&empty[s]);
        }
        if (!ok) break;
        tc_commit(&tfull[b]);
      }
      if (!ok) {
        abort_flag = 1;
        record_error(p.ctl, MOE_ERR_DEVICE_TIMEOUT, 0x200u);
      }
      // every MMA of this CTA is issued: let the next kernel's CTAs be
      // scheduled (they still wait for this grid to complete)
      pdl_trigger();
      // all MMAs issued by this thread complete before TMEM is released
      tc_commit(&done);
      mbar_wait_bounded(&done, 0, nullptr);
    }
  } else {
    // warps 2..9: quadrant q = warp % 4 (the TMEM lanes = tile rows this
    // warp may read), half h of the tile's output columns
    const int q = warp & 3;
    const int h = (warp - 2) >> 2;
    const int rr = q * 32 + lane;
    const int qbar = 1 + q;  // named barrier of the quadrant's two warps
    uint32_t tc = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++tc) {
      const TileInfo ti = decode(tile, n_tiles, tile_off, s_off, G);
      const uint32_t b = tc & 1, tph = (tc >> 1) & 1;
      bool got = mbar_wait_bounded(&tfull[b], tph, &abort_flag);
      // staged: the quadrant's two warps meet at named barriers below, so
      // they stop together (and this barrier also orders the previous
      // tile's copy-out before the staging rows are rewritten)
      if constexpr (STAGED) got = named_bar_and(qbar, 64, got);
      if (!got) {
        abort_flag = 1;
        record_error(p.ctl, MOE_ERR_DEVICE_TIMEOUT, 0x300u);
        break;
      }
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + b * ACC_STRIDE;
      const bool valid = rr < ti.rows;
      const int64_t grow = (int64_t)ti.row0 + rr;
      constexpr int OC = out_cols<BN, EPI>();
      constexpr int HC = OC / 2;
      static_assert(HC % 32 == 0, "each epilogue half covers whole 32-column groups");
      __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out) + grow * p.ld_out + ti.nt * OC;
      uint8_t* stg = sOut + (size_t)rr * staged_row_bytes<BN, EPI>();
      // 32 output columns per TMEM round trip: issue all loads, then wait once
#pragma unroll 1
      for (int c = h * HC; c < (h + 1) * HC; c += 32) {
        uint32_t pk[16];
        if constexpr (EPI == kEpiSwiGLU) {
          uint32_t g0[16], g1[16], u0[16], u1[16];
          tmem_ld16(taddr + c, g0);
          tmem_ld16(taddr + c + 16, g1);
          tmem_ld16(taddr + OC + c, u0);
          tmem_ld16(taddr + OC + c + 16, u1);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            pk[i] = pack_bf16x2(silu_mul(__uint_as_float(g0[2 * i]), __uint_as_float(u0[2 * i])),
                                silu_mul(__uint_as_float(g0[2 * i + 1]), __uint_as_float(u0[2 * i + 1])));
            pk[8 + i] = pack_bf16x2(silu_mul(__uint_as_float(g1[2 * i]), __uint_as_float(u1[2 * i])),
                                    silu_mul(__uint_as_float(g1[2 * i + 1]), __uint_as_float(u1[2 * i + 1])));
          }
        } else {
          uint32_t r0[16], r1[16];
          tmem_ld16(taddr + c, r0);
          tmem_ld16(taddr + c + 16, r1);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            pk[i] = pack_bf16x2(__uint_as_float(r0[2 * i]), __uint_as_float(r0[2 * i + 1]));
            pk[8 + i] = pack_bf16x2(__uint_as_float(r1[2 * i]), __uint_as_float(r1[2 * i + 1]));
          }
        }
        uint4* o = reinterpret_cast<uint4*>(STAGED ? static_cast<void*>(stg + c * 2)
                                                   : static_cast<void*>(out + c));
        if (!STAGED && valid && p.out_v8) {
          // whole 32-byte sectors: measured 3.5% fewer cycles per k-block
          // than 16-byte stores on the large workload's gate/up GEMM
          st_global_v8(o, pk);
          st_global_v8(o + 2, pk + 8);
        } else if (STAGED || valid) {
#pragma unroll
          for (int v = 0; v < 4; ++v) o[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
        }
      }
      if constexpr (STAGED) {
        // the accumulator is free once it is in shared memory
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[b]);
        named_bar_sync(qbar, 64);  // both halves of every row staged
        // copy-out: warp h writes rows [16h, 16h + 16) of the quadrant, whole
        // rows per instruction (16 bytes a lane), so every store covers full
        // contiguous row segments
        constexpr int RB = OC * 2;    // bytes of one output row of the tile
        constexpr int CPR = RB / 16;  // 16-byte chunks per row
        constexpr int RPI = 32 / CPR; // rows per warp instruction
        static_assert(CPR <= 32 && 32 % CPR == 0, "row chunks tile a warp");
        const int ch = lane % CPR;
#pragma unroll
        for (int r = q * 32 + h * 16 + lane / CPR; r < q * 32 + h * 16 + 16; r += RPI) {
          const uint4 v = *reinterpret_cast<const uint4*>(sOut + (size_t)r * staged_row_bytes<BN, EPI>() + ch * 16);
          if (r < ti.rows)
            *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) +
                                      ((int64_t)ti.row0 + r) * p.ld_out + ti.nt * OC + ch * 8) = v;
        }
        continue;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[b]);
    }
  }

  tc_fence_before();
  __syncwarp();  // role branches diverged single lanes: reconverge before the CTA barrier
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

}  // namespace

// ------------------------------------------------------------- host side
namespace {
PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

}  // namespace

// 2-D bf16 K-major operand [rows, K]: box of 64 K-elements (128 B) x box_rows,
// 128-byte swizzle, out-of-range rows read as zero
bool make_kmajor_map(CUtensorMap* m, const void* base, int64_t rows, int K, int box_rows) {
  auto enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)K * 2};
  cuuint32_t box[2] = {(cuuint32_t)BK, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
                   estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_f32_map(CUtensorMap* m, const void* base, int64_t rows, int cols, int box_rows) {
  auto enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)cols * 4};
  cuuint32_t box[2] = {32, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides, box,
                   estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

namespace {

template <int BN, int EPI, bool GATHER, bool STAGED>
cudaError_t run(const GemmArgs& a, cudaStream_t s) {
  constexpr size_t smem = smem_bytes_for<BN, EPI, STAGED, GATHER>();
  cudaError_t e = set_smem_limit((const void*)gemm_tc_kernel<BN, EPI, GATHER, STAGED>, smem);
  if (e != cudaSuccess) return e;
  CUtensorMap mA, mB;
  // gather mode reads A with cp.async; its tensor map is built but unused
  if (!make_kmajor_map(&mA, a.A, GATHER ? a.src_rows : a.rows, a.K, BM)) return cudaErrorInvalidValue;
  if (!make_kmajor_map(&mB, a.B, (int64_t)a.G * a.n_per_group, a.K, BN)) return cudaErrorInvalidValue;
  Params p;
  p.offsets = a.offsets;
  p.A = a.A;
  p.gather = a.gather;
  p.src_rows = a.src_rows;
  p.rows = a.rows;
  p.G = a.offsets ? a.G : 1;
  p.K = a.K;
  p.n_per_group = a.n_per_group;
  p.n_out = a.n_out;
  p.out = a.out;
  p.ld_out = a.ld_out;
  p.out_v8 = (reinterpret_cast<uintptr_t>(a.out) % 32 == 0) && ((a.ld_out * 2) % 32 == 0);
  p.ctl = a.ctl;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // upper bound of the tile count: every group adds at most one partial tile
  const int64_t mt_max = (a.rows + BM - 1) / BM + a.G;
  const int64_t tiles_max = mt_max * (a.n_per_group / BN);
  const int grid = (int)std::min<int64_t>(tiles_max, (int64_t)sms * ctas_per_sm<BN, STAGED, GATHER>());
  if (grid <= 0) return cudaSuccess;
  return launch_pdl(gemm_tc_kernel<BN, EPI, GATHER, STAGED>, dim3(grid), dim3(threads_for<GATHER>()), smem, s,
                    mA, mB, p);
}

}  // namespace

cudaError_t launch_gemm_tc(int epi, int bn, const GemmArgs& a, cudaStream_t s) {
  if (a.rows == 0) return cudaSuccess;
  const bool g = a.gather != nullptr;
  // short K loops: stage the epilogue through shared memory (see above).
  // Measured on B200: with 16-byte row stores a win up to 24 k-blocks for
  // the down GEMM (d-wide rows) and up to 8 for gate/up; with the 32-byte
  // stores (32-byte aligned outputs) the unstaged epilogue wins from 6
  // k-blocks up (forwards 1-4% faster with f = 384-1536, 2-7% with d = 384
  // and 512), staging only pays below (0.6-1.4% at f = 128 and 256)
  const bool v8 = (reinterpret_cast<uintptr_t>(a.out) % 32 == 0) && ((a.ld_out * 2) % 32 == 0);
  const bool st = a.K / BK <= (v8 ? 4 : (epi == kEpiBF16 ? 24 : 8));
#define MOE_GEMM_CASE(EPI, BN)                                                         \
  if (epi == EPI && bn == BN)                                                          \
    return g ? (st ? run<BN, EPI, true, true>(a, s) : run<BN, EPI, true, false>(a, s)) \
             : (st ? run<BN, EPI, false, true>(a, s) : run<BN, EPI, false, false>(a, s));
  MOE_GEMM_CASE(kEpiSwiGLU, 256)
  MOE_GEMM_CASE(kEpiSwiGLU, 128)
  if (g) return cudaErrorInvalidValue;  // gather is for the gate/up GEMM
#undef MOE_GEMM_CASE
#define MOE_GEMM_CASE(EPI, BN) \
  if (epi == EPI && bn == BN) return st ? run<BN, EPI, false, true>(a, s) : run<BN, EPI, false, false>(a, s);
  MOE_GEMM_CASE(kEpiBF16, 256)
  MOE_GEMM_CASE(kEpiBF16, 128)
  MOE_GEMM_CASE(kEpiBF16, 64)
#undef MOE_GEMM_CASE
  return cudaErrorInvalidValue;
}

}  // namespace moe
