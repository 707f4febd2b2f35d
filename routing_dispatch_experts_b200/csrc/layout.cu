// layout.cu - expert-grouped dispatch layout and the deduplicated send layout.
//
// Blocks of kTokPerBlock tokens (all k assignments of a token stay in one
// block), two phases:
//
//  1. histogram + decoupled lookback (lookback.cuh): each block counts its
//     assignments per expert, its distinct (token, rank) pairs per rank, and
//     two statistics, and obtains its exclusive prefix in every bin.  This
//     phase is either layout_hist_kernel below or the epilogue of the fused
//     router (route_tc.cu), which has the routing in registers already.
//  2. stable scatter: expert offsets from the totals, then every warp places
//     its contiguous run of assignments in flat-index order (match_any ranks
//     equal experts inside a 32-wide step), giving rows ordered by
//     (expert, t*k+j); send rows ordered by (rank, token) likewise, one per
//     distinct rank of a token.
//
// Deduplicated send layout: "Expert Coupling in MoE Pretraining", Abstract
// (each token is sent to each GPU once) and Table I (GPUs per token = distinct
// destinations; deduplication = rows removed as duplicates; the tokens split
// evenly over the GPUs give the home rank).
#include "lookback.cuh"

namespace moe {

namespace {

constexpr int kWarps = kLayoutThreads / 32;
constexpr int kTokPerWarp = kTokPerBlock / kWarps;
constexpr int kMaxIdx = kTokPerBlock * 16;  // the block's routing, staged in smem

struct Params {
  const int32_t* idx;
  int64_t T;
  int k, E, ep, nb, bins, stall_block;
  int64_t limit_ns;
  RankMap map;
  Control* ctl;
  uint64_t* status;  // [nb][bins] lookback words (histogram-kernel mode)
  int32_t* totals;   // [bins]   (histogram-kernel mode)
  const uint16_t* block_hist;  // [bins][hist_stride] per-block counts (fused-router mode)
  int hist_stride;
  LayoutOut out;
};

constexpr int kMaxK = 16;

__global__ void __launch_bounds__(kLayoutThreads) layout_hist_kernel(const __grid_constant__ Params p) {
  __shared__ int hist[kMaxBins];
  __shared__ int s_ticket;
  __shared__ uint8_t s_map[256];
  const int tid = threadIdx.x;
  for (int i = tid; i < p.bins; i += kLayoutThreads) hist[i] = 0;
  for (int i = tid; i < p.E; i += kLayoutThreads) s_map[i] = p.map.r[i];
  pdl_wait();
  if (tid == 0) s_ticket = (int)atomicAdd(&p.ctl->ticket, 1u);
  __syncthreads();
  const int b = s_ticket;
  if (b >= p.nb) {  // only if the workspace was not zeroed, or two calls share it at once
    if (tid == 0) record_error(p.ctl, MOE_ERR_WORKSPACE, (uint32_t)b);
    return;
  }
  const int64_t t0 = (int64_t)b * kTokPerBlock;
  const int64_t t1 = min(p.T, t0 + kTokPerBlock);
  const int sbin = p.E + (p.ep > 1 ? p.ep : 0);  // the two stat bins
  int single = 0, home = 0;
  for (int64_t t = t0 + tid; t < t1; t += kLayoutThreads) {
    int e[kMaxK];
    bool ok = true;
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) {
      e[j] = j < p.k ? __ldg(p.idx + t * p.k + j) : 0;
      if (j < p.k && (unsigned)e[j] >= (unsigned)p.E) {
        record_error(p.ctl, MOE_ERR_DEVICE_INDEX, (uint32_t)(t * p.k + j));
        ok = false;
      }
    }
    if (ok) count_token<kMaxK>(e, p.k, t, p.T, p.E, p.ep, s_map, hist, &single, &home);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    single += __shfl_xor_sync(0xffffffffu, single, off);
    home += __shfl_xor_sync(0xffffffffu, home, off);
  }
  if ((tid & 31) == 0) {
    atomicAdd(&hist[sbin], single);
    atomicAdd(&hist[sbin + 1], home);
  }
  __syncthreads();
  const bool publish = b != p.stall_block;
  for (int bin = tid; bin < p.bins; bin += kLayoutThreads) {
    uint32_t excl = 0;
    if (!lookback_bin(p.status, p.bins, b, bin, (uint32_t)hist[bin], publish, p.limit_ns, &excl)) {
      record_error(p.ctl, MOE_ERR_DEVICE_TIMEOUT, (uint32_t)b);
      continue;
    }
    if (b == p.nb - 1) p.totals[bin] = (int32_t)(excl + (uint32_t)hist[bin]);
  }
}

__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

__global__ void __launch_bounds__(kLayoutThreads) layout_scatter_kernel(const __grid_constant__ Params p) {
  __shared__ int s_off[kMaxBins + 2];  // expert offsets [E+1], then rank offsets [ep+1]
  __shared__ int wh[kWarps][kMaxBins];
  __shared__ int s_idx[kMaxIdx];
  __shared__ int s_pre[kMaxBins];  // this block's exclusive prefix per bin
  __shared__ int s_tot[kMaxBins];  // totals per bin
  __shared__ int s_ok;
  __shared__ uint8_t s_map[256];
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int b = blockIdx.x;
  const int E = p.E, ep = p.ep, k = p.k;
  const bool dedup = ep > 1;
  const int sbin = E + (dedup ? ep : 0);
  const int64_t tb0 = (int64_t)b * kTokPerBlock;
  const int ntok = (int)(p.T - tb0 < kTokPerBlock ? p.T - tb0 : kTokPerBlock);
  pdl_wait();

  if (tid == 0) s_ok = *reinterpret_cast<volatile uint32_t*>(&p.ctl->status) == MOE_OK;
  if (p.block_hist) {
    // fused-router mode: the kernel boundary already ordered every block's
    // histogram, so sum them directly.  block_hist is [bins][stride] of
    // 16-bit counts; one thread per bin reads its row with 16-byte loads (8
    // blocks each), 16 in flight at a time -- one round for up to 128
    // blocks -- and keeps the total and this block's exclusive prefix
    // (integer sums: exact)
    const int hs = p.hist_stride;
    for (int bin = tid; bin < p.bins; bin += kLayoutThreads) {
      const int4* row = reinterpret_cast<const int4*>(p.block_hist + (size_t)bin * hs);
      int tot = 0, pre = 0;
      for (int q8 = 0; q8 * 8 < p.nb; q8 += 16) {
        int4 v[16];
#pragma unroll
        for (int u = 0; u < 16; ++u)
          v[u] = (q8 + u) * 8 < p.nb ? __ldg(row + q8 + u) : make_int4(0, 0, 0, 0);
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          const int q = (q8 + u) * 8;
          const uint32_t w[4] = {(uint32_t)v[u].x, (uint32_t)v[u].y, (uint32_t)v[u].z, (uint32_t)v[u].w};
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const int cnt = (int)((w[c >> 1] >> (16 * (c & 1))) & 0xFFFFu);
            const int x = q + c < p.nb ? cnt : 0;  // entries past nb are padding
            tot += x;
            pre += q + c < b ? x : 0;
          }
        }
      }
      s_tot[bin] = tot;
      s_pre[bin] = pre;
    }
  } else {
    // histogram-kernel mode: this block's inclusive prefixes from its
    // lookback words, which are then zeroed for the next call (nothing else
    // reads them); block 0 resets the ticket counter.  The exclusive prefix
    // is the inclusive one minus the block's own count (below).
    uint64_t* words = p.status + (size_t)b * p.bins;
    for (int i = tid; i < p.bins; i += kLayoutThreads) {
      s_pre[i] = (int)(uint32_t)words[i];
      s_tot[i] = p.totals[i];
      words[i] = 0;
    }
    if (b == 0 && tid == 0) p.ctl->ticket = 0;
  }
  // the block's routing, read once (coalesced) into shared memory, and the
  // expert -> rank map
  for (int i = tid; i < ntok * k; i += kLayoutThreads) s_idx[i] = __ldg(p.idx + tb0 * k + i);
  if (dedup)
    for (int i = tid; i < E; i += kLayoutThreads) s_map[i] = p.map.r[i];
  for (int i = tid; i < kWarps * kMaxBins; i += kLayoutThreads) (&wh[0][0])[i] = 0;
  __syncthreads();
  // what is left is short: let the next kernel's CTAs be scheduled
  pdl_trigger();
  if (!s_ok) return;

  // exclusive scans of the expert totals and the rank totals (one warp each)
  if (warp < 2) {
    const int n = warp == 0 ? E : (dedup ? ep : 0);
    const int base_bin = warp == 0 ? 0 : E;
    int* dst = warp == 0 ? s_off : s_off + E + 1;
    if (n > 0) {
      int carry = 0;
      for (int c0 = 0; c0 < n; c0 += 32) {
        const int i = c0 + lane;
        const int v = i < n ? s_tot[base_bin + i] : 0;
        int incl = v;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const int o = __shfl_up_sync(0xffffffffu, incl, off);
          if (lane >= off) incl += o;
        }
        if (i < n) dst[i] = carry + incl - v;
        carry += __shfl_sync(0xffffffffu, incl, 31);
      }
      if (lane == 0) dst[n] = carry;
    }
  }
  // per-warp histograms of this block's assignments / send rows
  const int tw0 = min(ntok, warp * kTokPerWarp), tw1 = min(ntok, tw0 + kTokPerWarp);
  const int aw0 = tw0 * k, aw1 = tw1 * k;
  for (int a = aw0 + lane; a < aw1; a += 32) atomicAdd(&wh[warp][s_idx[a]], 1);
  if (dedup) {
    // one count per distinct rank of the token (ranks compared against the
    // token's earlier slots, in registers)
    for (int t = tw0 + lane; t < tw1; t += 32) {
      int rr[kMaxK];
#pragma unroll
      for (int j = 0; j < kMaxK; ++j) {
        if (j < k) {
          rr[j] = s_map[s_idx[t * k + j]];
          bool seen = false;
#pragma unroll
          for (int q = 0; q < j; ++q) seen |= rr[q] == rr[j];
          if (!seen) atomicAdd(&wh[warp][E + rr[j]], 1);
        }
      }
    }
  }
  __syncthreads();

  if (b == 0) {
    for (int e = tid; e < E; e += kLayoutThreads) {
      p.out.counts[e] = s_tot[e];
      p.out.offsets[e] = s_off[e];
    }
    if (tid == 0) p.out.offsets[E] = s_off[E];
    if (dedup) {
      for (int r = tid; r < ep; r += kLayoutThreads) {
        p.out.rank_counts[r] = s_tot[E + r];
        p.out.rank_offsets[r] = s_off[E + 1 + r];
      }
      if (tid == 0) p.out.rank_offsets[ep] = s_off[E + 1 + ep];
    }
    if (p.out.stats && warp == 0) {
      int mx = 0, mn = 0x7FFFFFFF;
      for (int e = lane; e < E; e += 32) {
        mx = max(mx, s_tot[e]);
        mn = min(mn, s_tot[e]);
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        mn = min(mn, __shfl_xor_sync(0xffffffffu, mn, off));
      }
      if (lane == 0) {
        moe_stats st;
        st.rows_sent = dedup ? (int64_t)s_off[E + 1 + ep] : 0;
        st.dup_removed = dedup ? p.T * k - st.rows_sent : 0;
        st.tokens_single_rank = s_tot[sbin];
        st.home_rank_rows = s_tot[sbin + 1];
        st.max_expert_rows = mx;
        st.min_expert_rows = E > 0 ? mn : 0;
        *p.out.stats = st;
      }
    }
  }

  // warp-exclusive starting rows: global offset + this block's exclusive
  // prefix + the counts of the block's earlier warps
  const int nbins_used = E + (dedup ? ep : 0);
  for (int bin = tid; bin < nbins_used; bin += kLayoutThreads) {
    int own = 0;
    if (!p.block_hist)
      for (int w = 0; w < kWarps; ++w) own += wh[w][bin];
    int run = (bin < E ? s_off[bin] : s_off[E + 1 + (bin - E)]) + s_pre[bin] - own;
    for (int w = 0; w < kWarps; ++w) {
      const int c = wh[w][bin];
      wh[w][bin] = run;
      run += c;
    }
  }
  __syncthreads();

  // stable scatter of the assignments, in flat-index order
  const uint32_t lt = lanemask_lt();
  for (int a0 = aw0; a0 < aw1; a0 += 32) {
    const int a = a0 + lane;
    const bool valid = a < aw1;
    const int e = valid ? s_idx[a] : -1;
    const uint32_t peers = __match_any_sync(0xffffffffu, e);
    if (valid) {
      const int row = wh[warp][e] + __popc(peers & lt);
      const int64_t ga = tb0 * k + a;
      p.out.row_token[row] = (int32_t)(ga / k);
      p.out.slot_row[ga] = row;
    }
    __syncwarp();
    if (valid && lane == __ffs(peers) - 1) wh[warp][e] += __popc(peers);
    __syncwarp();
  }

  // deduplicated send rows, tokens in order, one row per distinct rank
  if (dedup) {
    const int nw = (ep + 31) >> 5;
    for (int tt = tw0; tt < tw1; tt += 32) {
      const int t = tt + lane;
      const bool valid = t < tw1;
      int rr[kMaxK];
#pragma unroll
      for (int j = 0; j < kMaxK; ++j) rr[j] = (valid && j < k) ? (int)s_map[s_idx[t * k + j]] : -1;
      const int64_t gt = tb0 + t;
      for (int i = 0; i < nw; ++i) {
        // this lane's ranks in [32i, 32i + 32), then the warp's union
        uint32_t mi = 0;
#pragma unroll
        for (int j = 0; j < kMaxK; ++j)
          if (rr[j] >= 0 && (rr[j] >> 5) == i) mi |= 1u << (rr[j] & 31);
        uint32_t u = __reduce_or_sync(0xffffffffu, mi);
        while (u) {
          const int rb = __ffs(u) - 1;
          u &= u - 1;
          const int r = (i << 5) + rb;
          const bool has = (mi >> rb) & 1u;
          const uint32_t bal = __ballot_sync(0xffffffffu, has);
          if (has) {
            const int srow = wh[warp][E + r] + __popc(bal & lt);
            p.out.send_token[srow] = (int32_t)gt;
#pragma unroll
            for (int j = 0; j < kMaxK; ++j)
              if (rr[j] == r) p.out.slot_send_row[gt * k + j] = srow;
          }
          __syncwarp();
          if (lane == 0) wh[warp][E + r] += __popc(bal);
          __syncwarp();
        }
      }
    }
  }
}

Params make_params(const int32_t* idx, int64_t T, int k, int E, int ep, const RankMap& map,
                   const LayoutOut& out, Control* ctl, uint64_t* status_words, int32_t* totals,
                   int stall_block, int64_t limit_ns) {
  Params p;
  p.idx = idx;
  p.T = T;
  p.k = k;
  p.E = E;
  p.ep = ep;
  p.nb = layout_blocks(T);
  p.bins = layout_bins(E, ep);
  p.stall_block = stall_block;
  p.limit_ns = limit_ns;
  p.map = map;
  p.ctl = ctl;
  p.status = status_words;
  p.totals = totals;
  p.block_hist = nullptr;
  p.hist_stride = 0;
  p.out = out;
  return p;
}

cudaError_t empty_layout(int E, int ep, const LayoutOut& out, cudaStream_t s) {
  // no tokens: counts and offsets are all zero, no send rows
  cudaError_t err = cudaMemsetAsync(out.counts, 0, sizeof(int32_t) * E, s);
  if (err == cudaSuccess) err = cudaMemsetAsync(out.offsets, 0, sizeof(int32_t) * (E + 1), s);
  if (err == cudaSuccess && ep > 1) {
    err = cudaMemsetAsync(out.rank_counts, 0, sizeof(int32_t) * ep, s);
    if (err == cudaSuccess) err = cudaMemsetAsync(out.rank_offsets, 0, sizeof(int32_t) * (ep + 1), s);
  }
  if (err == cudaSuccess && out.stats) err = cudaMemsetAsync(out.stats, 0, sizeof(moe_stats), s);
  return err;
}

}  // namespace

cudaError_t launch_layout(const int32_t* idx, int64_t T, int k, int E, int ep, const RankMap& map,
                          const LayoutOut& out, Control* ctl, uint64_t* status_words,
                          int32_t* totals, int stall_block, int64_t limit_ns, cudaStream_t s) {
  if (T == 0) return empty_layout(E, ep, out, s);
  Params p = make_params(idx, T, k, E, ep, map, out, ctl, status_words, totals, stall_block,
                         limit_ns);
  cudaError_t err = launch_pdl(layout_hist_kernel, dim3(p.nb), dim3(kLayoutThreads), 0, s, p);
  if (err != cudaSuccess) return err;
  return launch_pdl(layout_scatter_kernel, dim3(p.nb), dim3(kLayoutThreads), 0, s, p);
}

cudaError_t launch_layout_scatter(const int32_t* idx, int64_t T, int k, int E, int ep,
                                  const RankMap& map, const LayoutOut& out, Control* ctl,
                                  const uint16_t* block_hist, cudaStream_t s) {
  if (T == 0) return empty_layout(E, ep, out, s);
  Params p = make_params(idx, T, k, E, ep, map, out, ctl, nullptr, nullptr, -1, 0);
  p.block_hist = block_hist;
  p.hist_stride = layout_hist_stride(p.nb);
  return launch_pdl(layout_scatter_kernel, dim3(p.nb), dim3(kLayoutThreads), 0, s, p);
}

}  // namespace moe
