// permute_combine.cu - the two data-movement steps around the experts.
//
//  permute: x_perm[r] = x[row_token[r]]  (dispatch of token rows to their
//           experts' contiguous row ranges; "Expert Coupling in MoE
//           Pretraining", Abstract: dispatch tokens to their experts)
//  combine: y[t] = sum_j gate[t,j] * y_perm[slot_row[t*k+j]]  (gather the
//           expert outputs back and weight them by the gates)
#include <algorithm>

#include "kernels.cuh"

namespace moe {

namespace {

// ---------------------------------------------------------------- permute
// TMA-staged ring for rows longer than 1 KB (and for the token-order
// variant).  One warp per CTA.  Rows move in groups of `rps` rows (one group fills a
// 16 KB shared-memory stage); lane i of the warp owns row i of every group.
// Lane i issues a TMA bulk load of its source row into the stage (completing
// on the stage's mbarrier), then, LOOKAHEAD groups later, a TMA bulk store of
// the staged row to its destination.  A lane reuses a stage region only after
// its own bulk store from that region has finished reading (bulk-group wait),
// so loads of group g+LOOKAHEAD overlap the stores of group g.
#ifndef MOE_PERM_STAGES
#define MOE_PERM_STAGES 4
#endif
#ifndef MOE_PERM_LOOKAHEAD
#define MOE_PERM_LOOKAHEAD 2
#endif
#ifndef MOE_PERM_STAGE_BYTES
#define MOE_PERM_STAGE_BYTES 16384
#endif
#ifndef MOE_PERM_CTAS
#define MOE_PERM_CTAS 3
#endif
constexpr int kPermStages = MOE_PERM_STAGES;
constexpr int kPermLookahead = MOE_PERM_LOOKAHEAD;
constexpr uint32_t kPermStageBytes = MOE_PERM_STAGE_BYTES;
constexpr int kPermCtasPerSm = MOE_PERM_CTAS;
static_assert(kPermLookahead < kPermStages, "lookahead must leave a stage to store from");

// BY_TOKEN = false: item r is x_perm row r, read from x[row_token[r]].
// BY_TOKEN = true:  item t is x row t, read once and written to its k rows
// x_perm[slot_row[t*k + j]] -- x streams through once, which keeps DRAM
// traffic at |x| + |x_perm| when x does not fit in L2.
template <bool BY_TOKEN>
__global__ void __launch_bounds__(32) permute_kernel(const uint8_t* __restrict__ x,
                                                     const int32_t* __restrict__ index,
                                                     uint8_t* __restrict__ x_perm, int64_t R,
                                                     int64_t T, int k, uint32_t row_bytes, int rps) {
  extern __shared__ __align__(128) uint8_t stage[];
  __shared__ __align__(8) uint64_t full[kPermStages];
  __shared__ int dst_rows[BY_TOKEN ? kPermStages : 1][BY_TOKEN ? 32 * 16 : 1];
  const int lane = threadIdx.x;
  if (lane == 0) {
    for (int s = 0; s < kPermStages; ++s) mbar_init(&full[s], 1);
    fence_barrier_init();
  }
  __syncwarp();
  pdl_wait();
  const int64_t items = BY_TOKEN ? T : R;
  const int64_t ngroups = (items + rps - 1) / rps;
  const int64_t nmine = ngroups > blockIdx.x ? (ngroups - blockIdx.x + gridDim.x - 1) / gridDim.x : 0;
  for (int64_t i = 0; i < nmine + kPermLookahead; ++i) {
    if (i < nmine) {
      const int s = (int)(i % kPermStages);
      const int64_t g = blockIdx.x + i * gridDim.x;
      const int64_t r0 = g * rps;
      const int n = (int)(items - r0 < rps ? items - r0 : rps);
      // this lane's stores of group i - kPermStages read the same region
      bulk_wait_read<kPermStages - kPermLookahead - 1>();
      if (lane == 0) mbar_arrive_expect_tx(&full[s], (uint32_t)n * row_bytes);
      __syncwarp();
      if (lane < n) {
        int64_t src;
        if constexpr (BY_TOKEN) {
          src = r0 + lane;
          for (int j = 0; j < k; ++j) {
            // an out-of-range row (malformed input) is skipped
            const int32_t d = __ldg(index + src * k + j);
            dst_rows[s][lane * 16 + j] = (d >= 0 && d < R) ? d : -1;
          }
        } else {
          // an out-of-range token (malformed input) reads row 0 instead of
          // faulting; the result is then unspecified, as documented
          src = __ldg(index + r0 + lane);
          if (src < 0 || src >= T) src = 0;
        }
        bulk_load(stage + (size_t)s * kPermStageBytes + (size_t)lane * row_bytes,
                  x + src * row_bytes, row_bytes, &full[s]);
      }
    }
    const int64_t j = i - kPermLookahead;
    if (j >= 0 && j < nmine) {
      const int s = (int)(j % kPermStages);
      const int64_t g = blockIdx.x + j * gridDim.x;
      const int64_t r0 = g * rps;
      const int n = (int)(items - r0 < rps ? items - r0 : rps);
      // the loads of a group complete on the stage barrier; bounded wait
      if (!mbar_wait_bounded(&full[s], (uint32_t)((j / kPermStages) & 1), nullptr)) {
        // never expected: a bulk load did not land within the limit
        break;
      }
      if (lane < n) {
        const uint8_t* src = stage + (size_t)s * kPermStageBytes + (size_t)lane * row_bytes;
        if constexpr (BY_TOKEN) {
          for (int q = 0; q < k; ++q) {
            const int d = dst_rows[s][lane * 16 + q];
            if (d >= 0) bulk_store(x_perm + (int64_t)d * row_bytes, src, row_bytes);
          }
        } else {
          bulk_store(x_perm + (r0 + lane) * row_bytes, src, row_bytes);
        }
      }
      bulk_commit();
    }
  }
  bulk_wait<0>();
}

// Register copy for short rows: each warp copies 32 16-byte vectors per
// item (an item is a row, or a 512-byte piece of a longer row), U items in
// flight per lane, loads all issued before the stores.
template <int U>
__global__ void __launch_bounds__(256) permute_vec_kernel(const uint4* __restrict__ x,
                                                          const int32_t* __restrict__ row_token,
                                                          uint4* __restrict__ x_perm, int64_t R,
                                                          int64_t T, int V) {
  const int lane = threadIdx.x & 31;
  pdl_wait();
  const int ipr = (V + 31) / 32;  // items per row
  const int64_t items = R * ipr;
  const int64_t warp0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t it0 = warp0 * U; it0 < items; it0 += nwarps * U) {
    uint4 v[U];
    int64_t dst[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t it = it0 + u;
      dst[u] = -1;
      if (it < items) {
        const int64_t r = it / ipr;
        const int c = (int)(it - r * ipr) * 32 + lane;
        if (c < V) {
          int64_t src = __ldg(row_token + r);
          if (src < 0 || src >= T) src = 0;
          v[u] = __ldg(x + src * V + c);
          dst[u] = r * V + c;
        }
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u)
      if (dst[u] >= 0) x_perm[dst[u]] = v[u];
  }
}

// ---------------------------------------------------------------- combine
// One thread per 16-byte output vector (8 bf16 or 4 fp32 of one token's
// row): it reads the token's k slot rows and gates, loads the k matching
// vectors of y_perm and sums gate * value in fp32 with j ascending, then
// rounds once.  Consecutive threads cover consecutive vectors of a row.
template <typename T>
struct Vec;
template <>
struct Vec<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ static void acc(float* a, const uint4& q, float g) {
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
struct Vec<float> {
  static constexpr int N = 4;
  __device__ static void acc(float* a, const uint4& q, float g) {
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

template <typename T, int VPT>
__global__ void __launch_bounds__(128) combine_kernel(const uint4* __restrict__ y_perm,
                                                      const int32_t* __restrict__ slot_row,
                                                      const float* __restrict__ gate,
                                                      uint4* __restrict__ y, int64_t Tn, int V,
                                                      int k) {
  pdl_wait();
  // thread item i: vectors [i*VPT, i*VPT + VPT) of the flattened [T, V]
  // output (V % VPT == 0, so they belong to one token); the token's slot
  // rows and gates are loaded once and every vector load is issued before
  // any is used
  const int64_t n = Tn * V / VPT;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = i * VPT / V;
    const int v = (int)(i * VPT - t * V);
    float a[VPT][Vec<T>::N];
#pragma unroll
    for (int u = 0; u < VPT; ++u)
#pragma unroll
      for (int q = 0; q < Vec<T>::N; ++q) a[u][q] = 0.f;
    int j = 0;
    for (; j + 4 <= k; j += 4) {
      uint4 q[4][VPT];
      float g[4];
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        int64_t row = __ldg(slot_row + t * k + j + w);
        if (row < 0 || row >= Tn * k) row = 0;
        g[w] = gate ? __ldg(gate + t * k + j + w) : 1.f;
#pragma unroll
        for (int u = 0; u < VPT; ++u) q[w][u] = __ldg(y_perm + row * V + v + u);
      }
#pragma unroll
      for (int w = 0; w < 4; ++w)
#pragma unroll
        for (int u = 0; u < VPT; ++u) Vec<T>::acc(a[u], q[w][u], g[w]);
    }
    for (; j < k; ++j) {
      int64_t row = __ldg(slot_row + t * k + j);
      if (row < 0 || row >= Tn * k) row = 0;
      const float g = gate ? __ldg(gate + t * k + j) : 1.f;
      uint4 q[VPT];
#pragma unroll
      for (int u = 0; u < VPT; ++u) q[u] = __ldg(y_perm + row * V + v + u);
#pragma unroll
      for (int u = 0; u < VPT; ++u) Vec<T>::acc(a[u], q[u], g);
    }
#pragma unroll
    for (int u = 0; u < VPT; ++u) y[i * VPT + u] = Vec<T>::pack(a[u]);
  }
}

}  // namespace

cudaError_t launch_permute(const void* x, const int32_t* row_token, const int32_t* slot_row,
                           void* x_perm, int64_t T, int k, uint32_t row_bytes, cudaStream_t s) {
  const int64_t R = T * k;
  if (R == 0) return cudaSuccess;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // Short rows (<= 1 KB): the register copy keeps more rows in flight than
  // the staged ring; longer rows go through the TMA-staged ring.
  if (!slot_row && row_bytes <= 1024) {
    constexpr int U = 4;
    const int V = (int)(row_bytes / 16);
    const int64_t items = R * ((V + 31) / 32);
    const int64_t warps = (items + U - 1) / U;
    const int grid = (int)std::min<int64_t>((warps + 7) / 8, (int64_t)sms * 8);
    return launch_pdl(permute_vec_kernel<U>, dim3(grid), dim3(256), 0, s,
                      static_cast<const uint4*>(x), row_token, static_cast<uint4*>(x_perm), R, T, V);
  }
  const int smem = kPermStages * (int)kPermStageBytes;
  const bool by_token = slot_row != nullptr;
  {
    cudaError_t e = set_smem_limit(by_token ? (const void*)permute_kernel<true>
                                            : (const void*)permute_kernel<false>,
                                   (size_t)smem);
    if (e != cudaSuccess) return e;
  }
  const int rps = (int)std::min<uint32_t>(32u, kPermStageBytes / row_bytes);
  const int64_t ngroups = ((by_token ? T : R) + rps - 1) / rps;
  const int grid = (int)std::min<int64_t>(ngroups, (int64_t)sms * kPermCtasPerSm);
  if (by_token)
    return launch_pdl(permute_kernel<true>, dim3(grid), dim3(32), (size_t)smem, s,
                      static_cast<const uint8_t*>(x), slot_row, static_cast<uint8_t*>(x_perm), R,
                      T, k, row_bytes, rps);
  return launch_pdl(permute_kernel<false>, dim3(grid), dim3(32), (size_t)smem, s,
                    static_cast<const uint8_t*>(x), row_token, static_cast<uint8_t*>(x_perm), R, T, k,
                    row_bytes, rps);
}

cudaError_t launch_combine(int dtype, const void* y_perm, const int32_t* slot_row,
                           const float* gate, void* y, int64_t T, int d, int k, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  const int esz = dtype == MOE_BF16 ? 2 : 4;
  const int V = d * esz / 16;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // two vectors per thread (d % 64 == 0, so every row has an even number of
  // 16-byte vectors): more loads in flight per thread and, for a
  // fine-grained batch, a grid that fits one wave
  // 128-thread CTAs (one warp per SM sub-partition): launched early, they fit
  // beside the preceding expert-FFN CTA, whose warps leave about one warp's
  // worth of registers free on each sub-partition
  if (V % 2 != 0) return cudaErrorInvalidValue;
  const int64_t n = T * V / 2;
  const int grid = (int)std::min<int64_t>((n + 127) / 128, (int64_t)sms * 16);
  if (dtype == MOE_BF16)
    return launch_pdl(combine_kernel<__nv_bfloat16, 2>, dim3(grid), dim3(128), 0, s,
                      static_cast<const uint4*>(y_perm), slot_row, gate, static_cast<uint4*>(y), T,
                      V, k);
  return launch_pdl(combine_kernel<float, 2>, dim3(grid), dim3(128), 0, s,
                    static_cast<const uint4*>(y_perm), slot_row, gate, static_cast<uint4*>(y), T, V,
                    k);
}

}  // namespace moe
