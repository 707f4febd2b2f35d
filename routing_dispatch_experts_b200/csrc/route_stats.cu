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

// Capacity: every expert serves its assignments in priority order -- every
// token's first choice before any token's second choice (choice rank j
// ascending), tokens in order within a rank -- and keeps the first `cap`.
// The position of assignment (t, j) to expert e in e's queue is
//   (assignments to e in the columns before j)
//   + (tokens before t whose column j holds e),
// a stable counting sort of each choice column.  Tokens are split into
// chunks of kCapTok; capacity_hist_kernel counts each chunk's assignments
// per (column, expert), capacity_rank_kernel turns the counts into each
// chunk's base per (column, expert) and ranks the chunk's tokens within it
// (warp match, then per-warp counts scanned in warp order).
constexpr int kCapTok = 1024;  // tokens per chunk = threads per block

__global__ void __launch_bounds__(kCapTok)
    capacity_hist_kernel(const int32_t* __restrict__ idx, int64_t T, int k, int E, int nbc,
                         int32_t* __restrict__ H, Control* ctl) {
  __shared__ int hist[16 * 256];
  pdl_wait();
  for (int i = threadIdx.x; i < k * E; i += kCapTok) hist[i] = 0;
  __syncthreads();
  const int64_t t = (int64_t)blockIdx.x * kCapTok + threadIdx.x;
  bool bad = false;
  if (t < T)
    for (int j = 0; j < k; ++j) {
      const int e = __ldg(idx + t * k + j);
      if (e < 0 || e >= E) bad = true;
      else atomicAdd(&hist[j * E + e], 1);
    }
  if (__syncthreads_or(bad) && threadIdx.x == 0) record_error(ctl, MOE_ERR_DEVICE_INDEX, 0x900u);
  // H[j][chunk][e]
  for (int i = threadIdx.x; i < k * E; i += kCapTok) {
    const int j = i / E, e = i - j * E;
    H[((int64_t)j * nbc + blockIdx.x) * E + e] = hist[i];
  }
}

__global__ void __launch_bounds__(kCapTok)
    capacity_rank_kernel(const int32_t* __restrict__ idx, int64_t T, int k, int E, int nbc,
                         const int32_t* __restrict__ H, int64_t cap,
                         const float* __restrict__ gate, int32_t* __restrict__ keep,
                         float* __restrict__ kept_gate) {
  extern __shared__ int cap_smem[];
  int* base = cap_smem;           // [k][E]: queue position of the chunk's first entry
  int* wc = cap_smem + k * E;     // [32][E] (first [k][E]: column totals)
  pdl_wait();
  const int b = blockIdx.x;
  for (int i = threadIdx.x; i < k * E; i += kCapTok) {
    const int j = i / E, e = i - j * E;
    const int32_t* h = H + (int64_t)j * nbc * E + e;
    int pre = 0, tot = 0;
    for (int c = 0; c < nbc; ++c) {
      const int v = __ldg(h + (int64_t)c * E);
      pre += c < b ? v : 0;
      tot += v;
    }
    base[i] = pre;
    wc[i] = tot;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += kCapTok) {
    int acc = 0;
    for (int j = 0; j < k; ++j) {
      base[j * E + e] += acc;
      acc += wc[j * E + e];
    }
  }
  __syncthreads();
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int64_t t = (int64_t)b * kCapTok + threadIdx.x;
  for (int j = 0; j < k; ++j) {
    for (int i = threadIdx.x; i < 32 * E; i += kCapTok) wc[i] = 0;
    __syncthreads();
    int e = -1;
    if (t < T) e = __ldg(idx + t * k + j);
    const bool valid = e >= 0 && e < E;
    // lanes holding the same expert; invalid entries match nobody
    const unsigned m = __match_any_sync(0xffffffffu, valid ? e : E + lane);
    const int rank = __popc(m & ((1u << lane) - 1u));
    if (valid && rank == 0) wc[w * E + e] = __popc(m);
    __syncthreads();
    for (int q = threadIdx.x; q < E; q += kCapTok) {  // exclusive scan over warps
      int acc = 0;
      for (int ww = 0; ww < 32; ++ww) {
        const int v = wc[ww * E + q];
        wc[ww * E + q] = acc;
        acc += v;
      }
    }
    __syncthreads();
    if (valid) {
      const int64_t a = t * k + j;
      const bool kept = (int64_t)base[j * E + e] + wc[w * E + e] + rank < cap;
      keep[a] = kept ? 1 : 0;
      if (kept_gate) kept_gate[a] = kept ? (gate ? gate[a] : 1.f) : 0.f;
    }
    __syncthreads();  // wc is cleared for the next column
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

size_t capacity_scratch_bytes(int64_t T, int k, int E) {
  return (size_t)k * (size_t)((T + kCapTok - 1) / kCapTok) * (size_t)E * 4;
}

cudaError_t launch_capacity_keep(const int32_t* idx, int64_t T, int k, int E, int64_t cap,
                                 const float* gate, int32_t* keep, float* kept_gate, int32_t* H,
                                 Control* ctl, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  const int nbc = (int)((T + kCapTok - 1) / kCapTok);
  cudaError_t e = launch_pdl(capacity_hist_kernel, dim3((unsigned)nbc), dim3(kCapTok), 0, s, idx,
                             T, k, E, nbc, H, ctl);
  if (e != cudaSuccess) return e;
  const size_t smem = (size_t)(k + 32) * E * 4;
  if ((e = set_smem_limit((const void*)capacity_rank_kernel, smem)) != cudaSuccess) return e;
  return launch_pdl(capacity_rank_kernel, dim3((unsigned)nbc), dim3(kCapTok), smem, s, idx, T, k,
                    E, nbc, (const int32_t*)H, cap, gate, keep, kept_gate);
}

}  // namespace moe
