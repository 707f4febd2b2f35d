// gemm_pair.cu - the grouped GEMM of gemm_tc.cu on CTA pairs: 256-row tiles
// computed by two SMs with one tcgen05.mma (cta_group::2).
//
// Same computation, same epilogues (SwiGLU for the gate/up projection,
// plain bf16 for the down projection: "Revisiting MoE and Dense
// Speed-Accuracy Comparisons", 2.1 Architecture) and the same summation
// order per output (K blocks ascending) as gemm_tc.cu, so the results are
// bit-identical.  What changes is who holds what:
//   - a cluster of two CTAs on neighbouring SMs takes a 256-row tile of one
//     group (rows [row0, row0 + 256) clipped to the group) and BN columns;
//     CTA r (r = 0, 1) loads rows row0 + 128 r .. + 127 of A and rows
//     brow + (BN/2) r .. + BN/2 - 1 of B into its OWN shared memory with
//     plain (non-multicast) TMA loads, both counted on CTA 0's full barrier;
//   - thread 0 of CTA 0's MMA warp issues tcgen05.mma.cta_group::2 (M 256,
//     N BN) for both; each CTA's tensor memory receives its 128 rows x BN;
//     tcgen05.commit with a two-CTA mask frees both CTAs' stages and hands
//     both CTAs' accumulators to their epilogues;
//   - each CTA's epilogue drains its own 128 rows and arrives on CTA 0's
//     accumulator-empty barrier.
// Per SM a k-block stage holds 16 KB of A and BN/2 x 64 x 2 bytes of B
// instead of the whole B tile, so more stages fit and each SM pulls half
// the B bytes through L2 per FLOP.
//
// Gather mode (the gate/up GEMM): the permute fused into the operand load.
// A row r of the tile is row gather[r] of the source (x), so x_perm is never
// written; each lane of the producer warp loads four of the CTA's 128 rows
// per k block with one TMA gather4 (rows picked by index, one-row box) into
// the same swizzled layout a tile load writes, counted on CTA 0's barrier.
//
// Every mbarrier wait is bounded (one second); a role that gives up records
// MOE_ERR_DEVICE_TIMEOUT and raises the abort flag in both CTAs.  The final
// cluster barrier cannot time out, so every path of every role reaches it.
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "kernels.cuh"

namespace moe {

namespace {

constexpr int BM = 128, BK = 64, PM = 2 * BM;  // rows per CTA, K block, rows per pair
constexpr int kEpiWarps = 8;
constexpr int kThreads = 64 + 32 * kEpiWarps;

struct Params {
  const int32_t* offsets;  // NULL: one group of `rows` rows
  const int32_t* gather;   // gather mode: A row r is source row gather[r]
  int64_t src_rows;        // gather mode: rows of the source
  int64_t rows;
  int G, K, n_per_group;
  void* out;
  int64_t ld_out;
  // 1: `out` and the row pitch are 32-byte aligned (32-byte epilogue stores)
  int out_v8;
  Control* ctl;
  // combine fused into the down GEMM's epilogue (see GemmArgs)
  void* y;
  const int32_t* row_token;
  const int32_t* slot_row;
  const float* gate;
  int k;
  int64_t T;
  uint32_t* arrive;
};

template <int BN, int EPI>
constexpr int out_cols() { return EPI == kEpiSwiGLU ? BN / 2 : BN; }
template <int BN, int EPI>
constexpr uint32_t staged_row_bytes() { return out_cols<BN, EPI>() * 2 + 16; }
template <int BN, int EPI, bool STAGED>
constexpr uint32_t staging_bytes() { return STAGED ? 128u * staged_row_bytes<BN, EPI>() : 0u; }
template <int BN>
constexpr uint32_t stage_bytes() { return BM * BK * 2 + (BN / 2) * BK * 2; }
template <int BN, int EPI, bool STAGED>
constexpr int stages_for() {
  constexpr uint32_t n = (220u * 1024u - staging_bytes<BN, EPI, STAGED>()) / stage_bytes<BN>();
  return n > 8 ? 8 : (n < 2 ? 2 : (int)n);
}
template <int BN, int EPI, bool STAGED>
constexpr size_t smem_bytes_for() {
  return (size_t)stages_for<BN, EPI, STAGED>() * stage_bytes<BN>() + staging_bytes<BN, EPI, STAGED>() +
         1024;
}

struct TileInfo {
  int g, row0, rows, nt;
};

// tile -> (group, first row of the pair tile, rows of the group left from
// there, N tile); tile_off[g] = first pair tile of group g
__device__ __forceinline__ TileInfo decode(int tile, int n_tiles, const int* tile_off,
                                           const int* s_off, int G) {
  TileInfo ti;
  const int mt = tile / n_tiles;
  ti.nt = tile - mt * n_tiles;
  int lo = 1, hi = G;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (tile_off[mid] > mt) hi = mid; else lo = mid + 1;
  }
  ti.g = lo - 1;
  ti.row0 = s_off[ti.g] + (mt - tile_off[ti.g]) * PM;
  ti.rows = min(PM, s_off[ti.g + 1] - ti.row0);
  return ti;
}

__device__ __forceinline__ float silu_mul(float g, float u) {
  return __fdividef(g, 1.f + __expf(-g)) * u;
}

template <int BN, int EPI, bool STAGED, bool GATHER>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ Params p) {
  constexpr int STAGES = stages_for<BN, EPI, STAGED>();
  constexpr uint32_t A_BYTES = BM * BK * 2;
  constexpr uint32_t B_BYTES = (BN / 2) * BK * 2;  // this CTA's half of the B tile
  constexpr uint32_t TMEM_COLS = 2 * BN;            // two accumulators of BN columns
  static_assert(TMEM_COLS <= 512, "two accumulators fit in tensor memory");
  constexpr uint32_t IDESC = idesc_bf16_f32(PM, BN);
  constexpr uint32_t PAIR_TX = 2 * (A_BYTES + B_BYTES);  // both CTAs' bytes per stage

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * A_BYTES;
  uint8_t* sOut = smem + STAGES * (A_BYTES + B_BYTES);

  __shared__ __align__(8) uint64_t full[STAGES], empty[STAGES], tfull[2], tempty[2], done;
  __shared__ uint32_t tmem_base_s;
  __shared__ int tile_off[257];
  __shared__ int s_off[257];
  __shared__ volatile int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int G = p.G;

  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);   // CTA 0's producer; both CTAs' bytes
      mbar_init(&empty[s], 1);  // CTA 0's MMA commit, sent to both CTAs
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 2 * kEpiWarps);  // both CTAs' epilogue warps (CTA 0's barrier)
    }
    mbar_init(&done, 1);
    fence_barrier_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  } else if (warp == 1) {
    tmem_alloc_pair(&tmem_base_s, TMEM_COLS);
    tmem_relinquish_pair();
  }
  __syncwarp();
  pdl_wait();
  for (int g = threadIdx.x; g <= G; g += kThreads)
    s_off[g] = p.offsets ? min(max(__ldg(p.offsets + g), 0), (int)p.rows) : (g == 0 ? 0 : (int)p.rows);
  __syncthreads();
  if (warp == 0) {
    int carry = 0;
    for (int g0 = 0; g0 < G; g0 += 32) {
      const int g = g0 + lane;
      const int v = g < G ? (max(s_off[g + 1] - s_off[g], 0) + PM - 1) / PM : 0;
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
  __syncwarp();
  __syncthreads();
  // both CTAs' barriers are initialised (and TMEM allocated) before either
  // CTA signals the other
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = tmem_base_s;
  const int n_tiles = p.n_per_group / BN;
  const int total = tile_off[G] * n_tiles;
  const int kblocks = p.K / BK;
  const int cluster = blockIdx.x >> 1, nclusters = gridDim.x >> 1;
  const uint32_t peer_abort = mapa_shared(const_cast<int*>(&abort_flag), rank ^ 1u);
  // stop both CTAs: every role of either CTA then leaves its loop
  auto abort_pair = [&](uint32_t detail) {
    abort_flag = 1;
    st_shared_cluster_u32(peer_abort, 1u);
    record_error(p.ctl, MOE_ERR_DEVICE_TIMEOUT, detail);
  };

  if (warp == 0 && GATHER) {
    // the source rows of this lane's four A rows of a tile (rows past the
    // end of the gather list read row 0; they are never stored)
    auto rows_of = [&](int tile, int32_t (&src)[4]) {
      const TileInfo t2 = decode(tile, n_tiles, tile_off, s_off, G);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int64_t r = (int64_t)t2.row0 + (int)rank * BM + 4 * lane + q;
        const int32_t v = r < p.rows ? __ldg(p.gather + r) : 0;
        src[q] = (v >= 0 && v < p.src_rows) ? v : 0;
      }
    };
    uint32_t it = 0;
    bool ok = true;
    int32_t src[4], nxt[4];
    if (cluster < total) rows_of(cluster, nxt);
    for (int tile = cluster; tile < total && ok; tile += nclusters) {
      const TileInfo ti = decode(tile, n_tiles, tile_off, s_off, G);
      const int brow = ti.g * p.n_per_group + ti.nt * BN + (int)rank * (BN / 2);
#pragma unroll
      for (int q = 0; q < 4; ++q) src[q] = nxt[q];
      // the next tile's indices load while this tile's rows stream
      if (tile + nclusters < total) rows_of(tile + nclusters, nxt);
      for (int kb = 0; kb < kblocks; ++kb, ++it) {
        const uint32_t s = it % STAGES, ph = (it / STAGES) & 1;
        int good = 1;
        if (lane == 0) good = mbar_wait_bounded_cluster(&empty[s], ph ^ 1, &abort_flag);
        good = __shfl_sync(0xffffffffu, good, 0);
        if (!good) {
          ok = false;
          break;
        }
        const uint32_t fbar = mapa_shared(&full[s], 0);
        if (lane == 0) {
          if (leader) mbar_arrive_expect_tx(&full[s], PAIR_TX);
          tma_load_2d_pair(sB + s * B_BYTES, &tmB, fbar, kb * BK, brow);
        }
        tma_gather4_pair(sA + s * A_BYTES + lane * 4 * (BK * 2), &tmA, fbar, kb * BK, src[0], src[1],
                         src[2], src[3]);
      }
    }
    if (lane == 0) {
      if (!ok) abort_pair(0x1100u);
      const uint32_t first = it > (uint32_t)STAGES ? it - STAGES : 0;
      for (uint32_t q = first; q < it; ++q)
        mbar_wait_bounded(&empty[q % STAGES], (q / STAGES) & 1, &abort_flag);
    }
  } else if (warp == 0) {
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int tile = cluster; tile < total && ok; tile += nclusters) {
        const TileInfo ti = decode(tile, n_tiles, tile_off, s_off, G);
        const int arow = ti.row0 + (int)rank * BM;  // past the group: not stored
        const int brow = ti.g * p.n_per_group + ti.nt * BN + (int)rank * (BN / 2);
        for (int kb = 0; kb < kblocks; ++kb, ++it) {
          const uint32_t s = it % STAGES, ph = (it / STAGES) & 1;
          if (!mbar_wait_bounded_cluster(&empty[s], ph ^ 1, &abort_flag, true)) {
            ok = false;
            break;
          }
          if (leader) mbar_arrive_expect_tx(&full[s], PAIR_TX);
          const uint32_t fbar = mapa_shared(&full[s], 0);
          tma_load_2d_pair(sA + s * A_BYTES, &tmA, fbar, kb * BK, arow);
          tma_load_2d_pair(sB + s * B_BYTES, &tmB, fbar, kb * BK, brow);
        }
      }
      if (!ok) abort_pair(0x1100u);
      // tail: every issued stage has been consumed by the MMAs (so its loads
      // have landed) before this CTA may leave
      const uint32_t first = it > (uint32_t)STAGES ? it - STAGES : 0;
      for (uint32_t q = first; q < it; ++q)
        mbar_wait_bounded(&empty[q % STAGES], (q / STAGES) & 1, &abort_flag);
    }
  } else if (warp == 1) {
    if (leader && lane == 0) {
      uint32_t it = 0, tc = 0;
      bool ok = true;
      for (int tile = cluster; tile < total && ok; tile += nclusters, ++tc) {
        const uint32_t b = tc & 1, tph = (tc >> 1) & 1;
        if (!mbar_wait_bounded_cluster(&tempty[b], tph ^ 1, &abort_flag, true)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + b * BN;
        for (int kb = 0; kb < kblocks; ++kb, ++it) {
          const uint32_t s = it % STAGES, ph = (it / STAGES) & 1;
          // producer and MMA thread sleep in their waits (mbar_try_wait_sleep)
          if (!mbar_wait_bounded_cluster(&full[s], ph, &abort_flag, true)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + s * A_BYTES);
          const uint32_t b0 = smem_u32(sB + s * B_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            tc_mma_f16_pair(d_tmem, smem_desc_k128(a0 + kk * 32), smem_desc_k128(b0 + kk * 32),
                            IDESC, (kb | kk) != 0);
          tc_commit_pair_mc(&empty[s], 0x3);
        }
        if (!ok) break;
        tc_commit_pair_mc(&tfull[b], 0x3);
      }
      if (!ok) abort_pair(0x1200u);
      pdl_trigger();
      // every MMA of the pair has completed (they read both CTAs' shared
      // memory and write both CTAs' tensor memory) before either CTA leaves
      tc_commit_pair_mc(&done, 0x1);
      mbar_wait_bounded(&done, 0, nullptr);
    } else if (!leader && lane == 0) {
      pdl_trigger();
    }
  } else {
    const int q = warp & 3;
    const int h = (warp - 2) >> 2;
    const int rr = q * 32 + lane;
    const int qbar = 1 + q;
    uint32_t tc = 0;
    for (int tile = cluster; tile < total; tile += nclusters, ++tc) {
      const TileInfo ti = decode(tile, n_tiles, tile_off, s_off, G);
      const uint32_t b = tc & 1, tph = (tc >> 1) & 1;
      bool got = mbar_wait_bounded_cluster(&tfull[b], tph, &abort_flag);
      // one decision per warp (the TMEM loads below are warp-collective),
      // and per quadrant pair when staged (they meet at named barriers)
      got = __all_sync(0xffffffffu, got);
      if constexpr (STAGED) got = named_bar_and(qbar, 64, got);
      if (!got) {
        if (lane == 0) abort_pair(0x1300u);
        break;
      }
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + b * BN;
      const int my_row0 = ti.row0 + (int)rank * BM;  // first row this CTA holds
      const int my_rows = ti.rows - (int)rank * BM;   // may be <= 0: nothing stored
      const bool valid = rr < my_rows;
      const int64_t grow = (int64_t)my_row0 + rr;
      constexpr int OC = out_cols<BN, EPI>();
      constexpr int HC = OC / 2;
      static_assert(HC % 32 == 0, "each epilogue half covers whole 32-column groups");
      __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out) + grow * p.ld_out + ti.nt * OC;
      uint8_t* stg = sOut + (size_t)rr * staged_row_bytes<BN, EPI>();
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
          // whole 32-byte sectors (as in the one-CTA engine)
          st_global_v8(o, pk);
          st_global_v8(o + 2, pk + 8);
        } else if (STAGED || valid) {
#pragma unroll
          for (int v = 0; v < 4; ++v) o[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
        }
      }
      // the accumulator is drained (into registers or staging): hand it back
      // to CTA 0's MMA thread
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(mapa_shared(&tempty[b], 0));
      if constexpr (STAGED) {
        named_bar_sync(qbar, 64);  // both halves of every row staged
        constexpr int RB = OC * 2;
        constexpr int CPR = RB / 16;
        constexpr int RPI = 32 / CPR;
        static_assert(CPR <= 32 && 32 % CPR == 0, "row chunks tile a warp");
        const int ch = lane % CPR;
#pragma unroll
        for (int r = q * 32 + h * 16 + lane / CPR; r < q * 32 + h * 16 + 16; r += RPI) {
          const uint4 v = *reinterpret_cast<const uint4*>(sOut + (size_t)r * staged_row_bytes<BN, EPI>() + ch * 16);
          if (r < my_rows)
            *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) +
                                      ((int64_t)my_row0 + r) * p.ld_out + ti.nt * OC + ch * 8) = v;
        }
        if constexpr (EPI == kEpiBF16 && CPR == 32) {
          if (p.y) {
            // The combine: this warp wrote rows q*32 + h*16 .. +15 of the
            // tile (whole OC-column segments).  One arrival per row on its
            // token's counter for this N tile, after the stores are visible
            // device-wide; the k-th arrival sums the token's k row segments
            // in slot order (their writers fenced before arriving).
            __threadfence();
            __syncwarp();  // every lane's stores fenced before any lane arrives
            const int r = q * 32 + h * 16 + (lane & 15);
            bool last = false;
            int tok = 0;
            if (lane < 16 && r < my_rows) {
              tok = __ldg(p.row_token + my_row0 + r);
              tok = (tok >= 0 && tok < p.T) ? tok : 0;
              const unsigned prev = atomicAdd(p.arrive + (int64_t)tok * n_tiles + ti.nt, 1u);
              last = prev == (unsigned)(p.k - 1);
            }
            unsigned todo = __ballot_sync(0xffffffffu, last);
            if (todo) __threadfence();
            while (todo) {
              const int src = __ffs(todo) - 1;
              todo &= todo - 1;
              const int64_t t = __shfl_sync(0xffffffffu, tok, src);
              float acc[8];
#pragma unroll
              for (int i = 0; i < 8; ++i) acc[i] = 0.f;
              const int64_t col = (int64_t)ti.nt * OC + lane * 8;  // 32 lanes x 8 columns
              for (int j = 0; j < p.k; ++j) {
                int64_t row = __ldg(p.slot_row + t * p.k + j);
                if (row < 0 || row >= p.rows) row = 0;
                const float g = p.gate ? __ldg(p.gate + t * p.k + j) : 1.f;
                // written by other CTAs of this grid: read through L2
                const uint4 v = __ldcg(reinterpret_cast<const uint4*>(
                    static_cast<const __nv_bfloat16*>(p.out) + row * p.ld_out + col));
                const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                  acc[2 * i] = fmaf(g, bf16_lo(w[i]), acc[2 * i]);
                  acc[2 * i + 1] = fmaf(g, bf16_hi(w[i]), acc[2 * i + 1]);
                }
              }
              *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.y) + t * p.ld_out + col) =
                  make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]),
                             pack_bf16x2(acc[4], acc[5]), pack_bf16x2(acc[6], acc[7]));
            }
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncwarp();
  __syncthreads();
  // neither CTA leaves (or frees tensor memory) while the pair's MMAs or the
  // peer's roles may still use its shared or tensor memory
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

template <int BN, int EPI, bool STAGED, bool GATHER>
cudaError_t run(const GemmArgs& a, cudaStream_t s) {
  auto kernel = gemm_pair_kernel<BN, EPI, STAGED, GATHER>;
  constexpr size_t smem = smem_bytes_for<BN, EPI, STAGED>();
  cudaError_t e = set_smem_limit((const void*)kernel, smem);
  if (e != cudaSuccess) return e;
  CUtensorMap mA, mB;
  // gather mode: the source rows one at a time (gather4 boxes are one row high)
  if (!make_kmajor_map(&mA, a.A, GATHER ? a.src_rows : a.rows, a.K, GATHER ? 1 : BM))
    return cudaErrorInvalidValue;
  if (!make_kmajor_map(&mB, a.B, (int64_t)a.G * a.n_per_group, a.K, BN / 2)) return cudaErrorInvalidValue;
  Params p;
  p.offsets = a.offsets;
  p.gather = a.gather;
  p.src_rows = a.src_rows;
  p.rows = a.rows;
  p.G = a.offsets ? a.G : 1;
  p.K = a.K;
  p.n_per_group = a.n_per_group;
  p.out = a.out;
  p.ld_out = a.ld_out;
  p.out_v8 = (reinterpret_cast<uintptr_t>(a.out) % 32 == 0) && ((a.ld_out * 2) % 32 == 0);
  p.ctl = a.ctl;
  p.y = a.y;
  p.row_token = a.row_token;
  p.slot_row = a.slot_row;
  p.gate = a.gate;
  p.k = a.k;
  p.T = a.T;
  p.arrive = a.arrive;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  // as many pairs as the device holds at once (one CTA per SM), at most one
  // per pair tile (every group adds at most one partial tile)
  static std::mutex mu;
  static int cached_dev = -1, cached_clusters = 0;
  int dev = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  int clusters = 0;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (cached_dev == dev) {
      clusters = cached_clusters;
    } else {
      int sms = 148;
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
      cfg.gridDim = dim3(2 * (sms / 2));
      if (cudaOccupancyMaxActiveClusters(&clusters, (void*)kernel, &cfg) != cudaSuccess || clusters <= 0)
        clusters = sms / 2 - 4;
      cudaGetLastError();  // a failed query leaves nothing behind
      cached_dev = dev;
      cached_clusters = clusters;
    }
  }
  const int64_t mt_max = (a.rows + PM - 1) / PM + a.G;
  const int64_t tiles_max = mt_max * (a.n_per_group / BN);
  const int grid_clusters = (int)std::min<int64_t>(tiles_max, clusters);
  if (grid_clusters <= 0) return cudaSuccess;
  cfg.gridDim = dim3(2 * grid_clusters);
  return cudaLaunchKernelEx(&cfg, kernel, mA, mB, p);
}

}  // namespace

bool gemm_pair_supported(int epi, int bn, const GemmArgs& a) {
  // the row gather is the gate/up GEMM's (SwiGLU epilogue)
  return bn == 256 && (epi == kEpiSwiGLU || (epi == kEpiBF16 && a.gather == nullptr)) &&
         a.n_per_group % bn == 0 && (a.gather == nullptr || a.src_rows > 0);
}

cudaError_t launch_gemm_pair(int epi, int bn, const GemmArgs& a, cudaStream_t s) {
  if (a.rows == 0) return cudaSuccess;
  if (!gemm_pair_supported(epi, bn, a)) return cudaErrorInvalidValue;
  // The bf16 (down) epilogue is staged only for the combine summed in it
  // (which needs whole staged rows): with 32-byte stores, the unstaged
  // epilogue's six ring stages beat the staged one's four on B200 (top-2 /
  // top-6 forwards 2.6-3% faster, large 1-2%).  A short gate/up K loop
  // stages, as in gemm_tc.cu.
  const bool st = epi == kEpiBF16 ? a.y != nullptr : a.K / BK <= 8;
  const bool g = a.gather != nullptr;
  if (epi == kEpiSwiGLU)
    return g ? (st ? run<256, kEpiSwiGLU, true, true>(a, s) : run<256, kEpiSwiGLU, false, true>(a, s))
             : (st ? run<256, kEpiSwiGLU, true, false>(a, s) : run<256, kEpiSwiGLU, false, false>(a, s));
  return st ? run<256, kEpiBF16, true, false>(a, s) : run<256, kEpiBF16, false, false>(a, s);
}

}  // namespace moe
