// route_stats.cu - router observability and expert capacity.
//
//  * router statistics ("MoE Pretraining: Parallelism Layout Changes the
//    Model, Not Quality", Finding 3: routing margin = gap between the k-th
//    and (k+1)-th scores over the spread of the token's scores, near-ties
//    are where routing flips; Practical Implications: log the near-tie share
//    and compare against a recorded routing table);
//  * expert capacity ("Revisiting MoE and Dense Speed-Accuracy Comparisons",
//    2.1: a capacity factor with top-2 routing): which assignments an expert
//    of limited capacity keeps.
#include "kernels.cuh"

namespace moe {

namespace {

constexpr int kStatsWarps = 8;

// One warp per token; lane l holds the keys of experts l, l+32, ...
// (key = logit, plus the selection bias when one is given, summed in fp32
// as the top-k kernels do).  The k-th and (k+1)-th largest keys come from
// k+1 rounds of the same (key desc, index asc) selection; as values they are
// the k-th and (k+1)-th order statistics whatever the tie-break.  The margin
// (sk - sk1) / (max - min) is taken in double from the fp32 keys, which the
// conversion represents exactly.
template <int VPL>
__global__ void __launch_bounds__(32 * kStatsWarps)
    router_stats_kernel(const float* __restrict__ logits, const float* __restrict__ sel_bias,
                        int64_t T, int E, int k, const int32_t* __restrict__ idx,
                        const int32_t* __restrict__ recorded, double threshold,
                        double* __restrict__ margin_out, unsigned long long* __restrict__ counts) {
  __shared__ unsigned long long part[kStatsWarps][4];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int64_t t = (int64_t)blockIdx.x * kStatsWarps + w;
  pdl_wait();
  unsigned near = 0, chg_tok = 0, chg_exp = 0, chg_slot = 0;
  if (t < T) {
    const float* row = logits + t * E;
    float key[VPL];
    float mx = -INFINITY, mn = INFINITY;
#pragma unroll
    for (int c = 0; c < VPL; ++c) {
      const int e = lane + 32 * c;
      key[c] = 0.f;
      if (e < E) {
        key[c] = __ldg(row + e);
        if (sel_bias) key[c] += __ldg(sel_bias + e);
        mx = fmaxf(mx, key[c]);
        mn = fminf(mn, key[c]);
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
    }
    double m = INFINITY;  // k == E: every expert is chosen, no margin
    if (k < E) {
      uint32_t taken = 0;
      float sk = 0.f, sk1 = 0.f;
      for (int j = 0; j <= k; ++j) {
        float bv = -INFINITY;
        int bi = 0x7FFFFFFF;
#pragma unroll
        for (int c = 0; c < VPL; ++c) {
          const int e = lane + 32 * c;
          if (e < E && !((taken >> c) & 1u) && (bi == 0x7FFFFFFF || key[c] > bv)) {
            bv = key[c];
            bi = e;
          }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
          const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
          const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
          if (ov > bv || (ov == bv && oi < bi)) {
            bv = ov;
            bi = oi;
          }
        }
        if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
        if (j == k - 1) sk = bv;
        if (j == k) sk1 = bv;
      }
      const double spread = (double)mx - (double)mn;
      m = spread > 0.0 ? ((double)sk - (double)sk1) / spread : 0.0;
    }
    if (lane == 0) {
      if (margin_out) margin_out[t] = m;
      near = m < threshold ? 1u : 0u;
    }
    if (recorded) {
      // lane j < k holds a = idx[t,j], b = recorded[t,j]; the experts
      // swapped are the distinct a's that the recorded row does not hold
      const int a = lane < k ? __ldg(idx + t * k + lane) : -1;
      const int b = lane < k ? __ldg(recorded + t * k + lane) : -2;
      bool in_b = false, seen = false;
      for (int q = 0; q < k; ++q) {
        const int bq = __shfl_sync(0xffffffffu, b, q);
        const int aq = __shfl_sync(0xffffffffu, a, q);
        in_b |= a == bq;
        seen |= q < lane && aq == a;
      }
      const bool swapped = lane < k && !in_b && !seen;
      chg_exp = __popc(__ballot_sync(0xffffffffu, swapped));
      chg_slot = __popc(__ballot_sync(0xffffffffu, lane < k && a != b));
      chg_tok = chg_exp > 0 ? 1u : 0u;
    }
  }
  if (lane == 0) {
    part[w][0] = near;
    part[w][1] = chg_tok;
    part[w][2] = chg_exp;
    part[w][3] = chg_slot;
  }
  __syncthreads();
  if (threadIdx.x < 4) {
    unsigned long long s = 0;
#pragma unroll
    for (int q = 0; q < kStatsWarps; ++q) s += part[q][threadIdx.x];
    if (s) atomicAdd(counts + 1 + threadIdx.x, s);  // integer sums: order-free
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) counts[0] = (unsigned long long)T;
}

// Capacity: one block per expert e.  The expert serves its assignments in
// priority order -- every token's first choice before any token's second
// choice (choice rank j ascending), tokens in order within a rank -- and
// keeps the first `cap`.  Pass 1 counts e's assignments in each choice
// column; pass 2 walks the tokens in chunks and ranks, for each column j,
// the chunk's assignments to e with a block-wide prefix count.  The routing
// is read token-major (coalesced) and staged in shared memory per chunk.
constexpr int kCapThreads = 256;

__device__ __forceinline__ int block_excl_scan(int flag, int* warp_sums, int* total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const unsigned bal = __ballot_sync(0xffffffffu, flag);
  const int pre = __popc(bal & ((1u << lane) - 1u));
  if (lane == 0) warp_sums[w] = __popc(bal);
  __syncthreads();
  int base = 0, tot = 0;
#pragma unroll
  for (int q = 0; q < kCapThreads / 32; ++q) {
    const int v = warp_sums[q];
    base += q < w ? v : 0;
    tot += v;
  }
  __syncthreads();  // warp_sums is reused by the next call
  *total = tot;
  return base + pre;
}

__global__ void __launch_bounds__(kCapThreads)
    capacity_keep_kernel(const int32_t* __restrict__ idx, int64_t T, int k, int E, int64_t cap,
                         const float* __restrict__ gate, int32_t* __restrict__ keep,
                         float* __restrict__ kept_gate, Control* ctl) {
  __shared__ int s_idx[kCapThreads * 16];
  __shared__ int warp_sums[kCapThreads / 32];
  __shared__ int col_total[16];
  const int e = blockIdx.x;
  pdl_wait();
  // pass 1: assignments to e in each choice column (and, in block 0, the
  // range check of every index)
  int cnt[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) cnt[j] = 0;
  bool bad = false;
  for (int64_t t = threadIdx.x; t < T; t += kCapThreads) {
#pragma unroll
    for (int j = 0; j < 16; ++j)
      if (j < k) {
        const int v = __ldg(idx + t * k + j);
        cnt[j] += v == e;
        bad |= v < 0 || v >= E;
      }
  }
  if (e == 0) {  // block-uniform: the whole block takes part in the vote
    if (__syncthreads_or(bad) && threadIdx.x == 0) record_error(ctl, MOE_ERR_DEVICE_INDEX, 0x900u);
  }
  if (threadIdx.x < 16) col_total[threadIdx.x] = 0;
  __syncthreads();
#pragma unroll
  for (int j = 0; j < 16; ++j)
    if (j < k) {
      int c = cnt[j];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) c += __shfl_xor_sync(0xffffffffu, c, off);
      if ((threadIdx.x & 31) == 0 && c) atomicAdd(&col_total[j], c);
    }
  __syncthreads();
  // kept so far in column j before the current chunk: the columns before j
  // in full, then column j up to the chunk
  int64_t before[16];
  {
    int64_t acc = 0;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      before[j] = acc;
      if (j < k) acc += col_total[j];
    }
  }
  // pass 2
  for (int64_t t0 = 0; t0 < T; t0 += kCapThreads) {
    const int n = (int)(T - t0 < kCapThreads ? T - t0 : kCapThreads);
    for (int i = threadIdx.x; i < n * k; i += kCapThreads) s_idx[i] = __ldg(idx + t0 * k + i);
    __syncthreads();
    const int r = threadIdx.x;  // token t0 + r
#pragma unroll
    for (int j = 0; j < 16; ++j)
      if (j < k) {
        const bool mine = r < n && s_idx[r * k + j] == e;
        int tot;
        const int pre = block_excl_scan(mine, warp_sums, &tot);
        if (mine) {
          const int64_t a = (t0 + r) * k + j;
          const bool kept = before[j] + pre < cap;
          keep[a] = kept ? 1 : 0;
          if (kept_gate) kept_gate[a] = kept ? (gate ? gate[a] : 1.f) : 0.f;
        }
        before[j] += tot;
      }
    __syncthreads();  // s_idx is refilled next chunk
  }
}

}  // namespace

cudaError_t launch_router_stats(const float* logits, const float* sel_bias, int64_t T, int E,
                                int k, const int32_t* idx, const int32_t* recorded,
                                double threshold, double* margin, unsigned long long* counts,
                                cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  const unsigned grid = (unsigned)((T + kStatsWarps - 1) / kStatsWarps);
  switch ((E + 31) / 32) {
#define MOE_STATS_CASE(N)                                                                   \
  case N:                                                                                   \
    return launch_pdl(router_stats_kernel<N>, dim3(grid), dim3(32 * kStatsWarps), 0, s,     \
                      logits, sel_bias, T, E, k, idx, recorded, threshold, margin, counts);
    MOE_STATS_CASE(1)
    MOE_STATS_CASE(2)
    MOE_STATS_CASE(3)
    MOE_STATS_CASE(4)
    MOE_STATS_CASE(5)
    MOE_STATS_CASE(6)
    MOE_STATS_CASE(7)
    MOE_STATS_CASE(8)
#undef MOE_STATS_CASE
    default:
      return cudaErrorInvalidValue;
  }
}

cudaError_t launch_capacity_keep(const int32_t* idx, int64_t T, int k, int E, int64_t cap,
                                 const float* gate, int32_t* keep, float* kept_gate, Control* ctl,
                                 cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  return launch_pdl(capacity_keep_kernel, dim3((unsigned)E), dim3(kCapThreads), 0, s, idx, T, k, E,
                    cap, gate, keep, kept_gate, ctl);
}

}  // namespace moe
