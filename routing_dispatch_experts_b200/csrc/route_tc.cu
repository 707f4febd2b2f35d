// route_tc.cu - the router in one tcgen05 kernel: logits GEMM, bias, top-k
// selection, softmax gates, and (for the forward) the per-tile dispatch
// histogram that the layout scatter turns into offsets.
//
// Top-k routing with softmax gates over the k ("MoE Pretraining: Parallelism
// Layout Changes the Model, Not Quality", Methodology: top-4 routing;
// "Revisiting MoE and Dense Speed-Accuracy Comparisons", 2.1: Top-K routing;
// router weights "ME", Table 1).
//
// One CTA per 128-token tile:
//   warp 0      TMA producer: x tile [128 x 64] and W_r^T tile [E16 x 64] per
//               k-block, 128-byte swizzle, a ring as deep as fits (all
//               k-blocks of d = 256 in flight)
//   warp 1      TMEM allocation; one lane issues tcgen05.mma 128 x E16 x 16
//   warps 2-9   epilogue, two threads per token row (each reads a half of
//               the row's E16 fp32 logits with tcgen05.ld): + bias, and a
//               running top-k kept sorted in registers (key: logit desc,
//               index asc; equal logits keep the lower index because only a
//               strictly larger logit moves an entry); the other half's
//               list is merged into the first's through shared memory;
//               gates exp(l_j - l_0) / sum_i.  The logits tile is staged in
//               the operand ring (idle once the accumulator is complete) and
//               leaves by TMA tiled stores (E % 32 == 0) or a coalesced copy.
// With the histogram on, each token adds its experts, distinct ranks and two
// statistics to a shared histogram that the CTA stores as its column of
// block_hist [bins][nb]; the scatter kernel (after the kernel boundary, so every row is
// complete) sums the rows into offsets and per-block prefixes.
#include <algorithm>

#include "lookback.cuh"  // count_token

namespace moe {

namespace {

constexpr int BM = 128, BK = 64;
// operand ring depth: as many k-blocks in flight as fit (all of them for
// d = 256), so a CTA streaming a tall x tile keeps enough bytes in flight;
// half of it when two CTAs share an SM
constexpr int kMaxStages = 8;
constexpr size_t kRingBudget = 200u * 1024u;
constexpr int kEpiWarps = 8;                     // kParts per TMEM lane quadrant (16 measured slower)
constexpr int kParts = kEpiWarps / 4;            // threads per token row

struct Params {
  int64_t T;
  int K, E, BN, k;
  const float* bias;
  const float* sel_bias;  // [E] or NULL: added for the choice of experts only
  float* logits;
  int32_t* idx;
  float* gate;
  Control* ctl;
  int hist, ep, nb, bins, hist_stride;
  int stages;
  // logits out of the staged tile: 2 = TMA tiled stores of 128-byte-swizzled
  // 32-column blocks, 1 = coalesced copy of padded rows, 0 = direct stores
  int logits_mode;
  uint32_t merge_off;     // shared-memory offset of the partial top-k lists
  uint32_t staged_bytes;  // shared-memory bytes of one staged logits tile
  int sms;                // SMs of the device
  RankMap map;
  uint16_t* block_hist;
};

// Top-k by sorting networks on (logit, expert) keys, ordered by logit
// descending, expert ascending among equal logits (the key is a strict total
// order: experts are distinct).  `a` beats `b` when its logit is larger, or
// equal (IEEE: -0.0 == +0.0) with a lower expert index.
__device__ __forceinline__ bool key_beats(float va, int ia, float vb, int ib) {
  return va > vb || (va == vb && ia < ib);
}

// compare-exchange: the winner of slots p and q ends in p
__device__ __forceinline__ void key_cx(float& vp, int& ip, float& vq, int& iq) {
  const bool sw = key_beats(vq, iq, vp, ip);
  const float tv = sw ? vq : vp;
  const int ti = sw ? iq : ip;
  vq = sw ? vp : vq;
  iq = sw ? ip : iq;
  vp = tv;
  ip = ti;
}

// bitonic sort of N (a power of two) keys into descending key order
template <int N>
__device__ __forceinline__ void key_sort(float (&v)[N], int (&ix)[N]) {
#pragma unroll
  for (int size = 2; size <= N; size <<= 1)
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1)
#pragma unroll
      for (int i = 0; i < N; ++i) {
        const int j = i ^ stride;
        if (j > i) {
          // descending runs where (i & size) == 0, so the last pass
          // (size == N) leaves the whole array descending
          if ((i & size) == 0)
            key_cx(v[i], ix[i], v[j], ix[j]);
          else
            key_cx(v[j], ix[j], v[i], ix[i]);
        }
      }
}

// (tv, ti) := the N best keys of the two descending lists (tv, ti) and
// (gv, gi), descending: the better of each pair tv[i], gv[N-1-i] forms a
// bitonic sequence holding exactly the N best, which a bitonic merge sorts
template <int N>
__device__ __forceinline__ void key_merge(float (&tv)[N], int (&ti)[N], const float (&gv)[N],
                                          const int (&gi)[N]) {
#pragma unroll
  for (int i = 0; i < N; ++i) {
    const bool g = key_beats(gv[N - 1 - i], gi[N - 1 - i], tv[i], ti[i]);
    tv[i] = g ? gv[N - 1 - i] : tv[i];
    ti[i] = g ? gi[N - 1 - i] : ti[i];
  }
#pragma unroll
  for (int stride = N >> 1; stride > 0; stride >>= 1)
#pragma unroll
    for (int i = 0; i < N; ++i)
      if ((i & stride) == 0) key_cx(tv[i], ti[i], tv[i + stride], ti[i + stride]);
}

// MT = 128-row tiles per CTA.  MT = 1 (two CTAs per SM, at most 102
// registers a thread): the layout scatter that follows is launched early and
// must fit on the SM beside this kernel's CTA (registers are split per SM
// sub-partition); when it could not, the forward measured 4.5 us slower.
// MT = 2 (one CTA per SM, when there are more tiles than SMs): both tiles'
// x blocks share each W_r block of the ring, so an SM keeps 128 KB of x in
// flight instead of 96 KB and reads W_r from L2 half as often; the
// epilogue has 16 warps (four per TMEM lane quadrant: two per tile).
template <int MT>
constexpr int route_threads() { return 64 + 32 * kEpiWarps * MT; }

template <int KMAX, int MT>
__global__ void __launch_bounds__(route_threads<MT>(), (MT == 1 ? 2 : 1))
    route_fused_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                       const __grid_constant__ CUtensorMap tmL, const __grid_constant__ Params p) {
  constexpr int EPI = kEpiWarps * MT;  // epilogue warps
  constexpr int NT = route_threads<MT>();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t A_BYTES = BM * BK * 2;  // one tile's x block
  const uint32_t B_BYTES = (uint32_t)p.BN * BK * 2;
  uint8_t* sA = smem;
  const int kStages = p.stages;
  uint8_t* sB = smem + kStages * MT * A_BYTES;

  __shared__ __align__(8) uint64_t full[kMaxStages], empty[kMaxStages], tfull;
  __shared__ uint32_t tmem_base_s;
  __shared__ int hist[MT][kMaxBins];
  __shared__ float s_bias[256];
  __shared__ float s_sbias[256];
  __shared__ uint8_t s_map[256];
  __shared__ volatile int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int acc_cols = MT * p.BN;
  const uint32_t tmem_cols = acc_cols <= 32 ? 32 : acc_cols <= 64 ? 64 : acc_cols <= 128 ? 128
                                                 : acc_cols <= 256 ? 256 : 512;

  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(&tfull, 1);
    fence_barrier_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    if (p.logits_mode == 2) tma_prefetch_desc(&tmL);
  }
  for (int i = threadIdx.x; i < MT * kMaxBins; i += NT) (&hist[0][0])[i] = 0;
  if (warp == 1) {
    tmem_alloc(&tmem_base_s, tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncwarp();  // role branches diverged single lanes: reconverge before the CTA barrier
  __syncthreads();
  tc_fence_after();
  pdl_wait();
  const uint32_t tmem_base = tmem_base_s;
  const int b0 = blockIdx.x * MT;  // first tile of this CTA
  const int ntiles = min(MT, p.nb - b0);
  const bool tile_ok = ntiles > 0;
  const int kblocks = p.K / BK;

  if (warp == 0) {
    if (lane == 0 && tile_ok) {
      int kb = 0;
      for (; kb < kblocks; ++kb) {
        const uint32_t s = kb % kStages, ph = (kb / kStages) & 1;
        if (!mbar_wait_bounded(&empty[s], ph ^ 1, &abort_flag)) {
          abort_flag = 1;
          record_error(p.ctl, MOE_ERR_DEVICE_TIMEOUT, 0x400u);
          break;
        }
        mbar_arrive_expect_tx(&full[s], ntiles * A_BYTES + B_BYTES);
        for (int m = 0; m < ntiles; ++m)
          tma_load_2d(sA + (s * MT + m) * A_BYTES, &tmA, &full[s], kb * BK, (int32_t)((b0 + m) * BM));
        tma_load_2d(sB + s * B_BYTES, &tmB, &full[s], kb * BK, 0);
      }
      for (int q = kb > kStages ? kb - kStages : 0; q < kb; ++q)  // drain
        mbar_wait_bounded(&full[q % kStages], (q / kStages) & 1, nullptr);
    }
  } else if (warp == 1) {
    if (lane == 0 && tile_ok) {
      const uint32_t idesc = idesc_bf16_f32(BM, p.BN);
      bool ok = true;
      for (int kb = 0; kb < kblocks; ++kb) {
        const uint32_t s = kb % kStages, ph = (kb / kStages) & 1;
        if (!mbar_wait_bounded(&full[s], ph, &abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t b_0 = smem_u32(sB + s * B_BYTES);
        for (int m = 0; m < ntiles; ++m) {
          const uint32_t a0 = smem_u32(sA + (s * MT + m) * A_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            tc_mma_f16(tmem_base + m * p.BN, smem_desc_k128(a0 + kk * 32),
                       smem_desc_k128(b_0 + kk * 32), idesc, (kb | kk) != 0);
        }
        tc_commit(&empty[s]);
      }
      if (!ok) {
        abort_flag = 1;
        record_error(p.ctl, MOE_ERR_DEVICE_TIMEOUT, 0x500u);
      }
      // arrives when every MMA above has completed (also on the error path)
      tc_commit(&tfull);
    }
  } else if (tile_ok) {
    // epilogue warp e: quadrant q = warp % 4 (the TMEM lanes it may read),
    // tile m and part (which share of the row's 16-column chunks it scans)
    const int q = warp & 3;
    const int grp = (warp - 2) >> 2;  // 0 .. kParts * MT - 1
    const int m = grp % MT;
    const int part = grp / MT;  // 0 .. kParts-1
    const int rr = q * 32 + lane;
    const bool tile_m = m < ntiles;
    const int64_t row0 = (int64_t)(b0 + m) * BM;
    const int64_t t = row0 + rr;
    const bool valid = tile_m && t < p.T;
    const int nchunks = p.BN / 16;
    const int per = (nchunks + kParts - 1) / kParts;
    const int c_lo = min(part * per, nchunks);
    const int c_hi = min(c_lo + per, nchunks);
    // bias and expert -> rank map in shared memory (read after the
    // predecessor's completion, like every input)
    for (int i = threadIdx.x - 64; i < p.E; i += 32 * EPI) {
      s_bias[i] = p.bias ? __ldg(p.bias + i) : 0.f;
      s_sbias[i] = p.sel_bias ? __ldg(p.sel_bias + i) : 0.f;
      s_map[i] = p.map.r[i];
    }
    const bool sel = p.sel_bias != nullptr;
    named_bar_sync(1, 32 * EPI);
    float tv[KMAX];
    int ti[KMAX];
#pragma unroll
    for (int s = 0; s < KMAX; ++s) {
      tv[s] = -INFINITY;
      ti[s] = 0x7FFFFFFF;
    }
    const bool have = mbar_wait_bounded(&tfull, 0, &abort_flag) && !abort_flag;
    // the rest of this CTA is short: let the next kernel's CTAs be scheduled
    pdl_trigger();
    // The logits tiles are staged in the operand ring (every MMA has
    // completed, so nothing reads it any more), tile m at staged_bytes * m.
    // Mode 2: 32-column blocks of 128 rows x 128 B, 16-byte chunk x of row r
    // at chunk x ^ (r % 8) (the 128-byte swizzle the tensor map undoes);
    // mode 1: rows of 4E + 16 bytes.
    const int mode = p.logits_mode;
    const uint32_t lstride = (uint32_t)p.E * 4 + 16;
    uint8_t* stile = smem + (size_t)m * p.staged_bytes;
    float* lrow = p.logits + t * p.E;
    if (have && tile_m) {
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + m * p.BN;
      for (int ch = c_lo; ch < c_hi; ++ch) {
        const int c = ch * 16;
        uint32_t r[16];
        tmem_ld16(taddr + c, r);
        tmem_ld_wait();
        float v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]) + (c + i < p.E ? s_bias[c + i] : 0.f);
        if (mode == 2) {
          // E % 32 == 0: the chunk's 16 columns are 4 whole 16-byte chunks
          uint8_t* blk = stile + (size_t)(c >> 5) * (BM * 128) + rr * 128;
          const int x0 = (c & 31) >> 2;
#pragma unroll
          for (int u = 0; u < 4; ++u)
            *reinterpret_cast<float4*>(blk + (((x0 + u) ^ (rr & 7)) << 4)) =
                make_float4(v[4 * u], v[4 * u + 1], v[4 * u + 2], v[4 * u + 3]);
        } else if (mode == 1) {
          float* srow = reinterpret_cast<float*>(stile + (size_t)rr * lstride);
          if (c + 16 <= p.E) {
#pragma unroll
            for (int i = 0; i < 16; i += 4)
              *reinterpret_cast<float4*>(srow + c + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
          } else {
#pragma unroll
            for (int i = 0; i < 16; ++i)
              if (c + i < p.E) srow[c + i] = v[i];
          }
        } else if (valid) {
#pragma unroll
          for (int i = 0; i < 16; ++i)
            if (c + i < p.E) lrow[c + i] = v[i];
        }
        // the key: the logit, plus the selection bias when there is one;
        // the chunk's 16 keys in groups of G are sorted and merged into the
        // running top-KMAX list (columns past E never win)
        constexpr int G = KMAX < 16 ? KMAX : 16;
#pragma unroll
        for (int g0 = 0; g0 < 16; g0 += G) {
          float gv[KMAX];
          int gi[KMAX];
#pragma unroll
          for (int i = 0; i < KMAX; ++i) {
            const int col = c + g0 + i;
            const bool in = i < G && col < p.E;
            gv[i] = in ? (sel ? v[g0 + i] + s_sbias[col] : v[g0 + i]) : -INFINITY;
            gi[i] = in ? col : 0x7FFFFFFF;
          }
          key_sort<KMAX>(gv, gi);
          key_merge<KMAX>(tv, ti, gv, gi);
        }
      }
    }
    // parts 1.. leave their lists for part 0 in shared memory:
    // [MT][kParts-1][BM][KMAX] values, then the same of indices
    float* m_v = reinterpret_cast<float*>(smem + p.merge_off);
    int* m_i = reinterpret_cast<int*>(smem + p.merge_off) + MT * (kParts - 1) * BM * KMAX;
    if (part > 0) {
#pragma unroll
      for (int j = 0; j < KMAX; ++j) {
        m_v[((m * (kParts - 1) + part - 1) * BM + rr) * KMAX + j] = tv[j];
        m_i[((m * (kParts - 1) + part - 1) * BM + rr) * KMAX + j] = ti[j];
      }
    }
    if (mode == 2) fence_proxy_async_shared();  // staged tiles -> TMA store
    named_bar_sync(1, 32 * EPI);                // epilogue warps only
    if (have && mode == 2) {
      if (threadIdx.x == 64) {
        // rows past T are outside the tensor map and are not written
        for (int mm = 0; mm < ntiles; ++mm)
          for (int bb = 0; bb < p.E / 32; ++bb)
            tma_store_2d(&tmL, smem + (size_t)mm * p.staged_bytes + (size_t)bb * (BM * 128), bb * 32,
                         (int32_t)((b0 + mm) * BM));
        bulk_commit();
      }
    } else if (have && mode == 1) {
      // each tile's valid logits rows are contiguous in global memory: the
      // epilogue warps copy them out in 16-byte chunks, fully coalesced
      const int cpr = p.E / 4;  // chunks per row
      for (int mm = 0; mm < ntiles; ++mm) {
        const int64_t r0 = (int64_t)(b0 + mm) * BM;
        const int nvalid = (int)(p.T - r0 < BM ? p.T - r0 : BM);
        float4* dst = reinterpret_cast<float4*>(p.logits + r0 * p.E);
        const uint8_t* src = smem + (size_t)mm * p.staged_bytes;
        for (int c = threadIdx.x - 64; c < nvalid * cpr; c += 32 * EPI) {
          const int r = c / cpr, cc = c - r * cpr;
          dst[c] = *reinterpret_cast<const float4*>(src + (size_t)r * lstride + cc * 16);
        }
      }
    }
    if (part == 0 && tile_m) {
      // merge the other parts' lists (the key order decides ties)
#pragma unroll 1
      for (int pp = 0; pp < kParts - 1; ++pp) {
        float gv[KMAX];
        int gi[KMAX];
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
          gv[j] = m_v[((m * (kParts - 1) + pp) * BM + rr) * KMAX + j];
          gi[j] = m_i[((m * (kParts - 1) + pp) * BM + rr) * KMAX + j];
        }
        key_merge<KMAX>(tv, ti, gv, gi);
      }
      if (have && valid) {
        if (sel) {
          // gates from the chosen experts' own logits, read back from the
          // staged tile (or, in mode 0, from this CTA's global stores; the
          // barrier above ordered them) in place of the biased keys
#pragma unroll
          for (int j = 0; j < KMAX; ++j)
            if (j < p.k) {
              const int col = ti[j];
              if (mode == 2)
                tv[j] = *reinterpret_cast<const float*>(
                    stile + (size_t)(col >> 5) * (BM * 128) + rr * 128 +
                    (((((col & 31) >> 2) ^ (rr & 7))) << 4) + (col & 3) * 4);
              else if (mode == 1)
                tv[j] = *reinterpret_cast<const float*>(stile + (size_t)rr * lstride + col * 4);
              else
                tv[j] = lrow[col];
            }
        }
        float ex[KMAX];
        float z = 0.f;
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
          ex[j] = j < p.k ? expf(tv[j] - tv[0]) : 0.f;
          z += ex[j];
        }
#pragma unroll
        for (int j = 0; j < KMAX; ++j)
          if (j < p.k) {
            p.idx[t * p.k + j] = ti[j];
            p.gate[t * p.k + j] = ex[j] / z;
          }
      }
      if (p.hist) {
        int single = 0, home = 0;
        if (have && valid) count_token<KMAX>(ti, p.k, t, p.T, p.E, p.ep, s_map, hist[m], &single, &home);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
          single += __shfl_xor_sync(0xffffffffu, single, off);
          home += __shfl_xor_sync(0xffffffffu, home, off);
        }
        const int sbin = p.E + (p.ep > 1 ? p.ep : 0);
        if (lane == 0) {
          atomicAdd(&hist[m][sbin], single);
          atomicAdd(&hist[m][sbin + 1], home);
        }
      }
    }
    // the staged tiles have been read by the TMA stores before the CTA exits
    if (have && mode == 2 && threadIdx.x == 64) bulk_wait_read<0>();
  }
  tc_fence_before();
  __syncwarp();  // role branches diverged single lanes: reconverge before the CTA barrier
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, tmem_cols);
  }
  if (p.hist)  // bin-major [bins][stride], so the scatter reads rows of blocks
    for (int mm = 0; mm < ntiles; ++mm)
      for (int bin = threadIdx.x; bin < p.bins; bin += NT)
        p.block_hist[(size_t)bin * p.hist_stride + b0 + mm] = (uint16_t)hist[mm][bin];
}

// shared-memory bytes the epilogue of MT tiles needs after the GEMM: the
// staged logits tiles and the partial top-k lists of the other parts
template <int KMAX, int MT>
size_t epilogue_bytes(const Params& p, uint32_t* staged_bytes) {
  const size_t staged = p.logits_mode == 2 ? (size_t)p.E * 512
                        : p.logits_mode == 1 ? (size_t)BM * (p.E * 4 + 16) : 0;
  const size_t sb = (staged + 1023) & ~size_t(1023);
  if (staged_bytes) *staged_bytes = (uint32_t)sb;
  return (size_t)MT * sb + (size_t)MT * (kParts - 1) * BM * KMAX * 8;
}

// The ring's stages for MT tiles per CTA and the dynamic shared memory they
// take; false when they do not fit next to the kernel's static arrays.
template <int KMAX, int MT>
bool plan_ring(Params& p, size_t* smem) {
  // the ring also holds, after the GEMM, the staged logits tiles and the
  // partial top-k lists of the other parts: grow it when they need more room
  const size_t stage = (size_t)MT * BM * BK * 2 + (size_t)p.BN * BK * 2;
  const size_t need = epilogue_bytes<KMAX, MT>(p, &p.staged_bytes);
  p.merge_off = (uint32_t)MT * p.staged_bytes;
  const size_t budget = MT == 1 && p.nb > p.sms ? kRingBudget / 2 : kRingBudget;
  int st = (int)(budget / stage);
  st = st > kMaxStages ? kMaxStages : st;
  st = st > p.K / BK ? p.K / BK : st;
  p.stages = st < 1 ? 1 : st;
  while ((size_t)p.stages * stage < need) ++p.stages;
  if (p.stages > kMaxStages) return false;
  *smem = (size_t)p.stages * stage + 1024;
  static size_t static_bytes = 0, optin = 0;
  if (optin == 0) {
    cudaFuncAttributes fa;
    int dev = 0, v = 0;
    cudaGetDevice(&dev);
    if (cudaFuncGetAttributes(&fa, (const void*)route_fused_kernel<KMAX, MT>) != cudaSuccess ||
        cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
      return false;
    static_bytes = fa.sharedSizeBytes;
    optin = (size_t)v;
  }
  return *smem + static_bytes <= optin;
}

template <int KMAX, int MT>
cudaError_t run(const RouteArgs& a, const CUtensorMap& mA, const CUtensorMap& mB,
                const CUtensorMap& mL, Params p, cudaStream_t s) {
  size_t smem = 0;
  if (!plan_ring<KMAX, MT>(p, &smem)) return cudaErrorInvalidValue;
  // dynamic shared memory grows with E; raise the kernel's limit when needed
  cudaError_t e = set_smem_limit((const void*)route_fused_kernel<KMAX, MT>, smem);
  if (e != cudaSuccess) return e;
  const unsigned grid = (unsigned)((p.nb + MT - 1) / MT);
  return launch_pdl(route_fused_kernel<KMAX, MT>, dim3(grid), dim3(route_threads<MT>()), smem, s,
                    mA, mB, mL, p);
}

template <int KMAX>
cudaError_t run_mt(const RouteArgs& a, const CUtensorMap& mA, const CUtensorMap& mB,
                   const CUtensorMap& mL, Params p, cudaStream_t s) {
  // two tiles per CTA when there are more tiles than SMs and both tiles'
  // accumulators fit in tensor memory, their epilogue in the ring budget and
  // the ring in shared memory
  if (p.nb > p.sms && 2 * p.BN <= 512 && epilogue_bytes<KMAX, 2>(p, nullptr) <= kRingBudget) {
    Params q = p;
    size_t smem = 0;
    if (plan_ring<KMAX, 2>(q, &smem)) return run<KMAX, 2>(a, mA, mB, mL, p, s);
  }
  return run<KMAX, 1>(a, mA, mB, mL, p, s);
}

}  // namespace

cudaError_t launch_route_tc(const RouteArgs& a, cudaStream_t s) {
  if (a.T == 0) return cudaSuccess;
  Params p;
  p.T = a.T;
  p.K = a.d;
  p.E = a.E;
  p.BN = (a.E + 15) / 16 * 16;
  p.k = a.k;
  p.bias = a.bias;
  p.sel_bias = a.sel_bias;
  p.logits = a.logits;
  p.idx = a.idx;
  p.gate = a.gate;
  p.ctl = a.ctl;
  p.hist = a.hist ? 1 : 0;
  p.ep = a.ep;
  p.nb = layout_blocks(a.T);
  p.bins = layout_bins(a.E, a.ep);
  p.hist_stride = layout_hist_stride(p.nb);
  {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    p.sms = sms;
  }
  p.map = a.map;
  p.block_hist = a.block_hist;
  CUtensorMap mA, mB, mL;
  if (!make_kmajor_map(&mA, a.x, a.T, a.d, BM)) return cudaErrorInvalidValue;
  if (!make_kmajor_map(&mB, a.wrT, p.BN, a.d, p.BN)) return cudaErrorInvalidValue;
  const bool al16 = (reinterpret_cast<uintptr_t>(a.logits) & 15) == 0;
  p.logits_mode = (al16 && a.E % 32 == 0) ? 2 : (al16 && a.E % 4 == 0) ? 1 : 0;
  if (p.logits_mode == 2 && !make_f32_map(&mL, a.logits, a.T, a.E, BM)) p.logits_mode = 1;
  if (p.logits_mode != 2) mL = mA;  // unused
  if (a.k <= 2) return run_mt<2>(a, mA, mB, mL, p, s);
  if (a.k <= 4) return run_mt<4>(a, mA, mB, mL, p, s);
  if (a.k <= 8) return run_mt<8>(a, mA, mB, mL, p, s);
  return run_mt<16>(a, mA, mB, mL, p, s);
}

}  // namespace moe
