// ep.cu - expert parallelism: the deduplicated dispatch of "Expert Coupling
// in MoE Pretraining" (Abstract: each token is sent to each GPU that holds
// one of its experts once, not once per expert; Table I: the rows removed;
// Fig. 7: baseline vs deduplicated dispatch) and its combine return path.
//
// One rank's forward over P ranks (tokens split over ranks, experts placed
// by the expert -> rank map):
//   1. router + dispatch layout with ep = P: the send plan (rank_counts,
//      send_token: one send row per (token, destination rank)),
//   2. ep_pack_kernel: the send rows, grouped by destination, each carrying
//      the token's row of x, its k gates and its k experts as the
//      destination's local expert ids (E/P for an expert held elsewhere),
//   3. the exchange (all-to-all of the send rows; outside this file),
//   4. on each rank, the expert FFN over the received rows' local experts
//      (layout over E/P + 1 groups, the last one collecting the "held
//      elsewhere" slots, which no GEMM reads), then
//      ep_partial_combine_kernel: one return row per received row, the
//      gated sum of that rank's experts for the token,
//   5. the reverse exchange, and ep_home_combine_kernel: each token's output
//      is the sum of its returned rows (one per distinct destination rank).
#include "kernels.cuh"

namespace moe {

namespace {

constexpr int kPackWarps = 8;

// The distinct send rows of token t, one per destination rank: lane j < k
// holds slot j's send row; the returned mask has bit j set for the first
// slot of each distinct, in-range row (the same in every lane).
__device__ __forceinline__ unsigned distinct_slots(const int32_t* __restrict__ slot_send_row,
                                                   int64_t t, int k, int64_t total, int lane,
                                                   int64_t* row_out) {
  int64_t s = -1;
  if (lane < k) s = __ldg(slot_send_row + t * k + lane);
  const bool ok = lane < k && s >= 0 && s < total;
  const unsigned m = __match_any_sync(0xffffffffu, ok ? (unsigned long long)s
                                                      : (unsigned long long)(-1 - lane));
  *row_out = s;
  return __ballot_sync(0xffffffffu, ok && (__ffs(m) - 1) == lane);
}

// One warp per token t: its distinct send rows (the distinct values of
// slot_send_row[t, :]); x[t] is read once, 32 x kPackU vectors at a time,
// and stored into each of them.  Send row s goes to the rank r with
// rank_offsets[r] <= s < rank_offsets[r+1] (binary search in shared
// memory).  It lands at row s of the send buffers (rows s >= cap are not
// stored) or, with `dests`, at row dests.d[r].row0 + s - rank_offsets[r]
// of rank r's receive buffers (the pack and the all-to-all in one pass:
// plain stores, to another GPU's memory through its peer mapping), rows
// past dests.d[r].rows not stored.
constexpr int kPackU = 4;
__global__ void __launch_bounds__(32 * kPackWarps)
    ep_pack_kernel(const uint4* __restrict__ x, int64_t T, int V, int k,
                   const int32_t* __restrict__ idx, const float* __restrict__ gate,
                   const int32_t* __restrict__ slot_send_row,
                   const int32_t* __restrict__ rank_offsets, int P, EpMaps maps, int E, int E_loc,
                   uint4* __restrict__ send_x, int32_t* __restrict__ send_idx,
                   float* __restrict__ send_gate, int64_t cap,
                   const __grid_constant__ EpDests dests, int use_dests) {
  __shared__ int s_off[257];
  pdl_wait();
  for (int i = threadIdx.x; i <= P; i += blockDim.x) s_off[i] = __ldg(rank_offsets + i);
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int64_t total = s_off[P];
  for (int64_t t = (int64_t)blockIdx.x * kPackWarps + (threadIdx.x >> 5); t < T;
       t += (int64_t)gridDim.x * kPackWarps) {
    int64_t s;
    const unsigned first = distinct_slots(slot_send_row, t, k, total, lane, &s);
    // lanes holding a distinct row: its rank, its row in the destination
    // buffers and their base pointers
    int r = 0;
    int64_t row = -1;
    uint4* dx = send_x;
    int32_t* di = send_idx;
    float* dg = send_gate;
    if ((first >> lane) & 1u) {
      int lo = 0, hi = P - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s_off[mid] <= s) lo = mid; else hi = mid - 1;
      }
      r = lo;
      if (use_dests) {
        const int64_t rel = s - s_off[r];
        if (rel < dests.d[r].rows) row = dests.d[r].row0 + rel;
        dx = static_cast<uint4*>(dests.d[r].recv_x);
        di = dests.d[r].recv_idx;
        dg = dests.d[r].recv_gate;
      } else if (s < cap) {
        row = s;
      }
    }
    const unsigned dm = __ballot_sync(0xffffffffu, row >= 0);
    if (dm == 0) continue;  // warp-uniform
    // the k local expert ids and gates of every stored row
    const int e = lane < k ? __ldg(idx + t * k + lane) : -1;
    const float g = lane < k ? (gate ? __ldg(gate + t * k + lane) : 1.f) : 0.f;
    for (unsigned b = dm; b; b &= b - 1) {
      const int d = __ffs(b) - 1;
      const int rd = __shfl_sync(0xffffffffu, r, d);
      const int64_t rowd = __shfl_sync(0xffffffffu, row, d);
      int32_t* dix = reinterpret_cast<int32_t*>(
          __shfl_sync(0xffffffffu, reinterpret_cast<unsigned long long>(di), d));
      float* dgx = reinterpret_cast<float*>(
          __shfl_sync(0xffffffffu, reinterpret_cast<unsigned long long>(dg), d));
      if (lane < k) {
        const bool here = e >= 0 && e < E && maps.rank[e] == rd;
        dix[rowd * k + lane] = here ? (int)maps.local[e] : E_loc;
        dgx[rowd * k + lane] = g;
      }
    }
    // this lane's destination row starts (lane d holds distinct row d's)
    uint4* dst_row = row >= 0 ? dx + row * V : nullptr;
    const uint4* src = x + t * V;
    for (int v0 = 0; v0 < V; v0 += 32 * kPackU) {
      uint4 q[kPackU];
#pragma unroll
      for (int u = 0; u < kPackU; ++u) {
        const int v = v0 + lane + 32 * u;
        if (v < V) q[u] = __ldg(src + v);
      }
      for (unsigned b = dm; b; b &= b - 1) {
        uint4* dst = reinterpret_cast<uint4*>(__shfl_sync(
            0xffffffffu, reinterpret_cast<unsigned long long>(dst_row), __ffs(b) - 1));
#pragma unroll
        for (int u = 0; u < kPackU; ++u) {
          const int v = v0 + lane + 32 * u;
          if (v < V) dst[v] = q[u];
        }
      }
    }
  }
}

template <typename T>
struct Acc;
template <>
struct Acc<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ static void add(float* a, const uint4& q, float g) {
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      a[2 * i] = fmaf(g, bf16_lo(w[i]), a[2 * i]);
      a[2 * i + 1] = fmaf(g, bf16_hi(w[i]), a[2 * i + 1]);
    }
  }
  __device__ static uint4 pack(const float* a) {
    return make_uint4(pack_bf16x2(a[0], a[1]), pack_bf16x2(a[2], a[3]), pack_bf16x2(a[4], a[5]),
                      pack_bf16x2(a[6], a[7]));
  }
};
template <>
struct Acc<float> {
  static constexpr int N = 4;
  __device__ static void add(float* a, const uint4& q, float g) {
    a[0] = fmaf(g, __uint_as_float(q.x), a[0]);
    a[1] = fmaf(g, __uint_as_float(q.y), a[1]);
    a[2] = fmaf(g, __uint_as_float(q.z), a[2]);
    a[3] = fmaf(g, __uint_as_float(q.w), a[3]);
  }
  __device__ static uint4 pack(const float* a) {
    return make_uint4(__float_as_uint(a[0]), __float_as_uint(a[1]), __float_as_uint(a[2]),
                      __float_as_uint(a[3]));
  }
};

// y_ret[i] = sum over slots j (ascending) of received row i whose expert is
// held here (local id < E_loc) of gate[i,j] * y_perm[slot_row[i*k + j]], in
// fp32, rounded once.  One warp per received row: lane j < k reads slot j,
// the local slots form a mask, then each lane sums kPartU of the row's
// vectors, four slots' loads in flight before they are added in slot order.
// With `rets`, received row t (from source rank s: rets.base[s] <= t <
// rets.base[s+1]) is stored at row rets.d[s].row0 + t - rets.base[s] of that
// source's return buffer instead of row t of y_ret.
constexpr int kPartWarps = 8, kPartU = 4;
template <typename T>
__global__ void __launch_bounds__(32 * kPartWarps)
    ep_partial_combine_kernel(const uint4* __restrict__ y_perm, const int32_t* __restrict__ slot_row,
                              const int32_t* __restrict__ recv_idx, const float* __restrict__ recv_gate,
                              int E_loc, uint4* __restrict__ y_ret, int64_t Tr, int V, int k,
                              const __grid_constant__ EpReturns rets, int use_rets) {
  pdl_wait();
  const int lane = threadIdx.x & 31;
  for (int64_t t = (int64_t)blockIdx.x * kPartWarps + (threadIdx.x >> 5); t < Tr;
       t += (int64_t)gridDim.x * kPartWarps) {
    const int e = lane < k ? __ldg(recv_idx + t * k + lane) : -1;
    const bool loc = lane < k && e >= 0 && e < E_loc;  // else held by another rank
    int64_t row = loc ? __ldg(slot_row + t * k + lane) : 0;
    if (row < 0 || row >= Tr * k) row = 0;
    const float g = loc ? __ldg(recv_gate + t * k + lane) : 0.f;
    const unsigned lm = __ballot_sync(0xffffffffu, loc);
    uint4* out = y_ret + t * V;
    if (use_rets) {
      // the source rank of received row t: last s with base[s] <= t
      int lo = 0, hi = rets.P - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (rets.base[mid] <= t) lo = mid; else hi = mid - 1;
      }
      out = static_cast<uint4*>(rets.d[lo].y_back) + (rets.d[lo].row0 + (t - rets.base[lo])) * V;
    }
    for (int v0 = 0; v0 < V; v0 += 32 * kPartU) {
      float a[kPartU][Acc<T>::N];
#pragma unroll
      for (int u = 0; u < kPartU; ++u)
#pragma unroll
        for (int q = 0; q < Acc<T>::N; ++q) a[u][q] = 0.f;
      unsigned b = lm;
      while (b) {  // warp-uniform
        uint4 q[4][kPartU];
        float gw[4];
        int n = 0;
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          const int d = b ? __ffs(b) - 1 : 0;
          const int64_t rd = __shfl_sync(0xffffffffu, row, d);
          gw[w] = __shfl_sync(0xffffffffu, g, d);
          const bool use = b != 0;
          b &= b - 1;
          n += use;
#pragma unroll
          for (int u = 0; u < kPartU; ++u) {
            const int v = v0 + lane + 32 * u;
            q[w][u] = use && v < V ? __ldg(y_perm + rd * V + v) : make_uint4(0, 0, 0, 0);
          }
        }
#pragma unroll
        for (int w = 0; w < 4; ++w)
          if (w < n)
#pragma unroll
            for (int u = 0; u < kPartU; ++u) Acc<T>::add(a[u], q[w][u], gw[w]);
      }
#pragma unroll
      for (int u = 0; u < kPartU; ++u) {
        const int v = v0 + lane + 32 * u;
        if (v < V) out[v] = Acc<T>::pack(a[u]);
      }
    }
  }
}

// y[t] = sum, over the distinct send rows of token t in slot order (each
// destination rank's row counted once), of y_back[row], in fp32, rounded
// once.  One warp per token: the distinct rows found once (distinct_slots),
// then each lane sums kHomeU of the row's vectors, four rows' loads in
// flight before they are added (in slot order).
constexpr int kHomeWarps = 8, kHomeU = 4;
template <typename T>
__global__ void __launch_bounds__(32 * kHomeWarps)
    ep_home_combine_kernel(const uint4* __restrict__ y_back, const int32_t* __restrict__ slot_send_row,
                           uint4* __restrict__ y, int64_t Tn, int V, int k, int64_t rows) {
  pdl_wait();
  const int lane = threadIdx.x & 31;
  for (int64_t t = (int64_t)blockIdx.x * kHomeWarps + (threadIdx.x >> 5); t < Tn;
       t += (int64_t)gridDim.x * kHomeWarps) {
    int64_t s;
    const unsigned dm = distinct_slots(slot_send_row, t, k, rows, lane, &s);
    for (int v0 = 0; v0 < V; v0 += 32 * kHomeU) {
      float a[kHomeU][Acc<T>::N];
#pragma unroll
      for (int u = 0; u < kHomeU; ++u)
#pragma unroll
        for (int q = 0; q < Acc<T>::N; ++q) a[u][q] = 0.f;
      unsigned b = dm;
      while (b) {  // warp-uniform
        uint4 q[4][kHomeU];
        int n = 0;
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          const int d = b ? __ffs(b) - 1 : 0;
          const int64_t row = __shfl_sync(0xffffffffu, s, d);
          const bool use = b != 0;
          b &= b - 1;
          n += use;
#pragma unroll
          for (int u = 0; u < kHomeU; ++u) {
            const int v = v0 + lane + 32 * u;
            q[w][u] = use && v < V ? __ldg(y_back + row * V + v) : make_uint4(0, 0, 0, 0);
          }
        }
#pragma unroll
        for (int w = 0; w < 4; ++w)
          if (w < n)
#pragma unroll
            for (int u = 0; u < kHomeU; ++u) Acc<T>::add(a[u], q[w][u], 1.f);
      }
#pragma unroll
      for (int u = 0; u < kHomeU; ++u) {
        const int v = v0 + lane + 32 * u;
        if (v < V) y[t * V + v] = Acc<T>::pack(a[u]);
      }
    }
  }
}

int grid_for(int64_t items, int per_block) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return (int)std::min<int64_t>((items + per_block - 1) / per_block, (int64_t)sms * 8);
}

// The ranks' rendezvous around a peer-memory exchange: rank `me` stores
// `epoch` into slot `me` of every rank's flag array (a release at system
// scope, after everything earlier in this stream, so the rows this rank
// stored into peers' buffers are visible before the flag is), then waits
// until every slot of its own array holds at least `epoch` (an acquire at
// system scope), giving up after wait_ns and recording
// MOE_ERR_DEVICE_TIMEOUT with detail = the first missing rank.
__global__ void ep_signal_wait_kernel(const __grid_constant__ EpFlags fl, int me, int P,
                                      uint64_t epoch, int64_t wait_ns, Control* ctl) {
  pdl_wait();
  const int r = threadIdx.x;
  if (r < P) {
    uint64_t* slot = fl.flags[r] + me;
    asm volatile("fence.acq_rel.sys;" ::: "memory");
    asm volatile("st.release.sys.global.u64 [%0], %1;" ::"l"(slot), "l"(epoch) : "memory");
  }
  __syncthreads();
  if (r < P) {
    const uint64_t* mine = fl.flags[me] + r;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
      uint64_t v;
      asm volatile("ld.acquire.sys.global.u64 %0, [%1];" : "=l"(v) : "l"(mine) : "memory");
      if (v >= epoch) break;
      if (globaltimer_ns() - t0 > (uint64_t)wait_ns) {
        record_error(ctl, MOE_ERR_DEVICE_TIMEOUT, (uint32_t)r);
        break;
      }
    }
  }
}

}  // namespace

cudaError_t launch_ep_pack(int dtype, const void* x, int64_t T, int d, int k, const int32_t* idx,
                           const float* gate, const int32_t* slot_send_row,
                           const int32_t* rank_offsets, int P, const EpMaps& maps, int E,
                           void* send_x, int32_t* send_idx, float* send_gate, int64_t cap,
                           const EpDests* dests, cudaStream_t s) {
  if (T == 0 || cap == 0) return cudaSuccess;
  const int V = d * (dtype == MOE_BF16 ? 2 : 4) / 16;
  const int grid = std::max(1, grid_for(T, kPackWarps));
  EpDests dd{};
  if (dests) dd = *dests;
  return launch_pdl(ep_pack_kernel, dim3(grid), dim3(32 * kPackWarps), 0, s,
                    static_cast<const uint4*>(x), T, V, k, idx, gate, slot_send_row, rank_offsets, P,
                    maps, E, E / P, static_cast<uint4*>(send_x), send_idx, send_gate, cap, dd,
                    dests ? 1 : 0);
}

cudaError_t launch_ep_partial_combine(int dtype, const void* y_perm, const int32_t* slot_row,
                                      const int32_t* recv_idx, const float* recv_gate, int E_loc,
                                      void* y_ret, int64_t Tr, int d, int k, const EpReturns* rets,
                                      cudaStream_t s) {
  if (Tr == 0) return cudaSuccess;
  const int V = d * (dtype == MOE_BF16 ? 2 : 4) / 16;
  const int grid = std::max(1, grid_for(Tr, kPartWarps));
  EpReturns rr{};
  if (rets) rr = *rets;
  const int use = rets ? 1 : 0;
  if (dtype == MOE_BF16)
    return launch_pdl(ep_partial_combine_kernel<__nv_bfloat16>, dim3(grid), dim3(32 * kPartWarps),
                      0, s, static_cast<const uint4*>(y_perm), slot_row, recv_idx, recv_gate, E_loc,
                      static_cast<uint4*>(y_ret), Tr, V, k, rr, use);
  return launch_pdl(ep_partial_combine_kernel<float>, dim3(grid), dim3(32 * kPartWarps), 0, s,
                    static_cast<const uint4*>(y_perm), slot_row, recv_idx, recv_gate, E_loc,
                    static_cast<uint4*>(y_ret), Tr, V, k, rr, use);
}

cudaError_t launch_ep_home_combine(int dtype, const void* y_back, const int32_t* slot_send_row,
                                   void* y, int64_t T, int d, int k, int64_t rows, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  const int V = d * (dtype == MOE_BF16 ? 2 : 4) / 16;
  const int grid = std::max(1, grid_for(T, kHomeWarps));
  if (dtype == MOE_BF16)
    return launch_pdl(ep_home_combine_kernel<__nv_bfloat16>, dim3(grid), dim3(32 * kHomeWarps), 0,
                      s, static_cast<const uint4*>(y_back), slot_send_row, static_cast<uint4*>(y), T,
                      V, k, rows);
  return launch_pdl(ep_home_combine_kernel<float>, dim3(grid), dim3(32 * kHomeWarps), 0, s,
                    static_cast<const uint4*>(y_back), slot_send_row, static_cast<uint4*>(y), T, V, k,
                    rows);
}

cudaError_t launch_ep_signal_wait(const EpFlags& fl, int me, int P, uint64_t epoch,
                                  int64_t wait_ns, Control* ctl, cudaStream_t s) {
  return launch_pdl(ep_signal_wait_kernel, dim3(1), dim3(256), 0, s, fl, me, P, epoch, wait_ns,
                    ctl);
}

}  // namespace moe
