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
constexpr int kThreads = 64 + 32 * kEpiWarps;    // producer + MMA + epilogue

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
  uint32_t merge_off;  // shared-memory offset of the partial top-k lists
  RankMap map;
  uint16_t* block_hist;
};

// insert (v, e) into the descending list (tv, ti); e arrives in increasing
// order, so an equal logit never displaces an earlier (lower) index
template <int KMAX>
__device__ __forceinline__ void topk_insert(float (&tv)[KMAX], int (&ti)[KMAX], float v, int e) {
#pragma unroll
  for (int s = KMAX - 1; s > 0; --s) {
    const bool above = v > tv[s - 1];
    const bool here = v > tv[s];
    tv[s] = above ? tv[s - 1] : (here ? v : tv[s]);
    ti[s] = above ? ti[s - 1] : (here ? e : ti[s]);
  }
  if (v > tv[0]) {
    tv[0] = v;
    ti[0] = e;
  }
}

// At most 102 registers a thread (two CTAs' worth): the layout scatter that
// follows is launched early and must fit on the SM beside this kernel's CTA
// (registers are split per SM sub-partition); when it could not, the forward
// measured 4.5 us slower.
template <int KMAX>
__global__ void __launch_bounds__(kThreads, 2)
    route_fused_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                       const __grid_constant__ CUtensorMap tmL, const __grid_constant__ Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t A_BYTES = BM * BK * 2;
  const uint32_t B_BYTES = (uint32_t)p.BN * BK * 2;
  uint8_t* sA = smem;
  const int kStages = p.stages;
  uint8_t* sB = smem + kStages * A_BYTES;

  __shared__ __align__(8) uint64_t full[kMaxStages], empty[kMaxStages], tfull;
  __shared__ uint32_t tmem_base_s;
  __shared__ int hist[kMaxBins];
  __shared__ float s_bias[256];
  __shared__ float s_sbias[256];
  __shared__ uint8_t s_map[256];
  __shared__ volatile int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t tmem_cols = p.BN <= 32 ? 32 : (p.BN <= 64 ? 64 : (p.BN <= 128 ? 128 : 256));

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
  for (int i = threadIdx.x; i < p.bins; i += kThreads) hist[i] = 0;
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
  const int b = blockIdx.x;
  const bool tile_ok = b < p.nb;
  const int64_t row0 = (int64_t)b * BM;
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
        mbar_arrive_expect_tx(&full[s], A_BYTES + B_BYTES);
        tma_load_2d(sA + s * A_BYTES, &tmA, &full[s], kb * BK, (int32_t)row0);
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
        const uint32_t a0 = smem_u32(sA + s * A_BYTES);
        const uint32_t b0 = smem_u32(sB + s * B_BYTES);
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk)
          tc_mma_f16(tmem_base, smem_desc_k128(a0 + kk * 32), smem_desc_k128(b0 + kk * 32), idesc,
                     (kb | kk) != 0);
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
    // warps 2..: quadrant q = warp % 4 (the TMEM lanes this warp may read),
    // part = which share of the row's 16-column chunks it scans
    const int q = warp & 3;
    const int part = (warp - 2) >> 2;  // 0 .. kParts-1
    const int rr = q * 32 + lane;
    const int64_t t = row0 + rr;
    const bool valid = t < p.T;
    const int nchunks = p.BN / 16;
    const int per = (nchunks + kParts - 1) / kParts;
    const int c_lo = min(part * per, nchunks);
    const int c_hi = min(c_lo + per, nchunks);
    // bias and expert -> rank map in shared memory (read after the
    // predecessor's completion, like every input)
    for (int i = threadIdx.x - 64; i < p.E; i += 32 * kEpiWarps) {
      s_bias[i] = p.bias ? __ldg(p.bias + i) : 0.f;
      s_sbias[i] = p.sel_bias ? __ldg(p.sel_bias + i) : 0.f;
      s_map[i] = p.map.r[i];
    }
    const bool sel = p.sel_bias != nullptr;
    named_bar_sync(1, 32 * kEpiWarps);
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
    // The logits tile is staged in the operand ring (every MMA has completed,
    // so nothing reads it any more).  Mode 2: 32-column blocks of 128 rows x
    // 128 B, 16-byte chunk x of row r at chunk x ^ (r % 8) (the 128-byte
    // swizzle the tensor map undoes); mode 1: rows of 4E + 16 bytes.
    const int mode = p.logits_mode;
    const uint32_t lstride = (uint32_t)p.E * 4 + 16;
    float* lrow = p.logits + t * p.E;
    if (have) {
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16);
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
          uint8_t* blk = smem + (size_t)(c >> 5) * (BM * 128) + rr * 128;
          const int x0 = (c & 31) >> 2;
#pragma unroll
          for (int u = 0; u < 4; ++u)
            *reinterpret_cast<float4*>(blk + (((x0 + u) ^ (rr & 7)) << 4)) =
                make_float4(v[4 * u], v[4 * u + 1], v[4 * u + 2], v[4 * u + 3]);
        } else if (mode == 1) {
          float* srow = reinterpret_cast<float*>(smem + (size_t)rr * lstride);
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
        // the key: the logit, plus the selection bias when there is one
#pragma unroll
        for (int i = 0; i < 16; ++i)
          if (c + i < p.E) topk_insert<KMAX>(tv, ti, sel ? v[i] + s_sbias[c + i] : v[i], c + i);
      }
    }
    // parts 1.. leave their lists for part 0 in shared memory
    float* m_v = reinterpret_cast<float*>(smem + p.merge_off);  // [kParts-1][BM][KMAX]
    int* m_i = reinterpret_cast<int*>(smem + p.merge_off) + (kParts - 1) * BM * KMAX;
    if (part > 0) {
#pragma unroll
      for (int j = 0; j < KMAX; ++j) {
        m_v[((part - 1) * BM + rr) * KMAX + j] = tv[j];
        m_i[((part - 1) * BM + rr) * KMAX + j] = ti[j];
      }
    }
    if (mode == 2) fence_proxy_async_shared();  // staged tile -> TMA store
    named_bar_sync(1, 32 * kEpiWarps);          // epilogue warps only
    if (have && mode == 2) {
      if (threadIdx.x == 64) {
        // rows past T are outside the tensor map and are not written
        for (int b = 0; b < p.E / 32; ++b)
          tma_store_2d(&tmL, smem + (size_t)b * (BM * 128), b * 32, (int32_t)row0);
        bulk_commit();
      }
    } else if (have && mode == 1) {
      // the tile's valid logits rows are contiguous in global memory: the
      // epilogue warps copy them out in 16-byte chunks, fully coalesced
      const int cpr = p.E / 4;  // chunks per row
      const int nvalid = (int)(p.T - row0 < BM ? p.T - row0 : BM);
      float4* dst = reinterpret_cast<float4*>(p.logits + row0 * p.E);
      for (int c = threadIdx.x - 64; c < nvalid * cpr; c += 32 * kEpiWarps) {
        const int r = c / cpr, cc = c - r * cpr;
        dst[c] = *reinterpret_cast<const float4*>(smem + (size_t)r * lstride + cc * 16);
      }
    }
    if (part == 0) {
      // later parts' columns are all higher, so inserting their entries part
      // by part, in list order, keeps lower indices first among equal logits
#pragma unroll 1
      for (int pp = 0; pp < kParts - 1; ++pp)
#pragma unroll
        for (int j = 0; j < KMAX; ++j)
          topk_insert<KMAX>(tv, ti, m_v[(pp * BM + rr) * KMAX + j], m_i[(pp * BM + rr) * KMAX + j]);
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
                    smem + (size_t)(col >> 5) * (BM * 128) + rr * 128 +
                    (((((col & 31) >> 2) ^ (rr & 7))) << 4) + (col & 3) * 4);
              else if (mode == 1)
                tv[j] = *reinterpret_cast<const float*>(smem + (size_t)rr * lstride + col * 4);
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
        if (have && valid) count_token<KMAX>(ti, p.k, t, p.T, p.E, p.ep, s_map, hist, &single, &home);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
          single += __shfl_xor_sync(0xffffffffu, single, off);
          home += __shfl_xor_sync(0xffffffffu, home, off);
        }
        const int sbin = p.E + (p.ep > 1 ? p.ep : 0);
        if (lane == 0) {
          atomicAdd(&hist[sbin], single);
          atomicAdd(&hist[sbin + 1], home);
        }
      }
    }
    // the staged tile has been read by the TMA stores before the CTA exits
    if (have && mode == 2 && threadIdx.x == 64) bulk_wait_read<0>();
  }
  tc_fence_before();
  __syncwarp();  // role branches diverged single lanes: reconverge before the CTA barrier
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, tmem_cols);
  }
  if (p.hist && tile_ok)  // bin-major [bins][stride], so the scatter reads rows of blocks
    for (int bin = threadIdx.x; bin < p.bins; bin += kThreads)
      p.block_hist[(size_t)bin * p.hist_stride + b] = (uint16_t)hist[bin];
}

template <int KMAX>
cudaError_t run(const RouteArgs& a, const CUtensorMap& mA, const CUtensorMap& mB,
                const CUtensorMap& mL, Params p, cudaStream_t s) {
  // the ring also holds, after the GEMM, the staged logits tile and the
  // partial top-k lists of parts 1-3: grow it when they need more room
  const size_t stage = (size_t)BM * BK * 2 + (size_t)p.BN * BK * 2;
  const size_t staged = p.logits_mode == 2 ? (size_t)p.E * 512
                        : p.logits_mode == 1 ? (size_t)BM * (p.E * 4 + 16) : 0;
  p.merge_off = (uint32_t)((staged + 15) & ~size_t(15));
  const size_t need = p.merge_off + (size_t)(kParts - 1) * BM * KMAX * 8;
  while ((size_t)p.stages * stage < need) ++p.stages;
  if (p.stages > kMaxStages) return cudaErrorInvalidValue;
  // dynamic shared memory grows with E; raise the kernel's limit when needed
  const size_t smem = (size_t)p.stages * stage + 1024;
  cudaError_t e = set_smem_limit((const void*)route_fused_kernel<KMAX>, smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(route_fused_kernel<KMAX>, dim3(p.nb), dim3(kThreads), smem, s, mA, mB, mL, p);
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
    // More tiles than SMs: a half-size ring lets two CTAs share an SM, so
    // every tile is resident at once instead of a second wave of tiles
    // starting when the first has finished (T = 32768, d = 4096, E = 128:
    // 74 us instead of 86 us; the bytes in flight per SM are unchanged).
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const size_t budget = p.nb > sms ? kRingBudget / 2 : kRingBudget;
    const size_t stage = (size_t)BM * BK * 2 + (size_t)p.BN * BK * 2;
    const int kblocks = a.d / BK;
    int st = (int)(budget / stage);
    st = st > kMaxStages ? kMaxStages : st;
    st = st > kblocks ? kblocks : st;
    p.stages = st < 1 ? 1 : st;
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
  if (a.k <= 2) return run<2>(a, mA, mB, mL, p, s);
  if (a.k <= 4) return run<4>(a, mA, mB, mL, p, s);
  if (a.k <= 8) return run<8>(a, mA, mB, mL, p, s);
  return run<16>(a, mA, mB, mL, p, s);
}

}  // namespace moe
