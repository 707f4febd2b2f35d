// route.cu - top-k expert selection with softmax gates, and the fp32 router.
//
// Top-k routing with softmax gates renormalised over the k ("MoE Pretraining:
// Parallelism Layout Changes the Model, Not Quality", Methodology / Models
// and Data: top-4 routing; "Revisiting MoE and Dense Speed-Accuracy
// Comparisons", 2.1 Architecture: Top-K routing).
#include "kernels.cuh"

namespace moe {

// One warp per token.  Lane l holds logits e = l, l+32, ... (VPL of them) in
// registers.  k rounds: every lane proposes its best remaining expert under
// the key (logit desc, index asc); a butterfly of shuffles finds the warp's
// best; its owner marks it taken.  The key is a total order, so every lane
// ends each round with the same winner.  Equal logits (-0.0 == +0.0 too)
// resolve to the lower index because the comparison is the IEEE one.
// Gates: softmax of the chosen logits, exp(l_j - l_0) / sum_i exp(l_i - l_0),
// the sum reduced by the same butterfly in every lane (deterministic).
// With a selection bias b[E] the experts are chosen on the fp32 sum l + b
// and the gates still come from the chosen experts' l (the auxiliary-loss-
// free router of "Expert Coupling in MoE Pretraining", Fig. 11: a per-expert
// bias steers which experts are picked, not how their outputs are weighted).
template <int VPL>
__global__ void __launch_bounds__(256) topk_kernel(const float* __restrict__ logits,
                                                   const float* __restrict__ sel_bias, int64_t T,
                                                   int E, int k, int32_t* __restrict__ idx,
                                                   float* __restrict__ gate) {
  const int lane = threadIdx.x & 31;
  const int64_t t = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  pdl_wait();
  if (t >= T) return;  // uniform per warp
  const float* row = logits + t * E;
  float v[VPL], key[VPL];
#pragma unroll
  for (int c = 0; c < VPL; ++c) {
    const int e = lane + 32 * c;
    v[c] = e < E ? __ldg(row + e) : 0.f;
    key[c] = (sel_bias && e < E) ? v[c] + __ldg(sel_bias + e) : v[c];
  }
  uint32_t taken = 0;
  float my_l = 0.f;
  int my_e = 0;
  for (int j = 0; j < k; ++j) {
    float bv = -INFINITY;
    int bi = 0x7FFFFFFF;
#pragma unroll
    for (int c = 0; c < VPL; ++c) {
      const int e = lane + 32 * c;
      if (e < E && !((taken >> c) & 1u)) {
        if (bi == 0x7FFFFFFF || key[c] > bv) {  // e ascending: keep the first of equals
          bv = key[c];
          bi = e;
        }
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
    // the winner's own logit (equal to its key without a selection bias),
    // from the lane that holds it
    float mine = 0.f;
#pragma unroll
    for (int c = 0; c < VPL; ++c)
      if (c == (bi >> 5)) mine = v[c];
    const float raw = __shfl_sync(0xffffffffu, mine, bi & 31);
    if (lane == j) {
      my_l = raw;
      my_e = bi;
    }
  }
  const float l0 = __shfl_sync(0xffffffffu, my_l, 0);
  float ex = lane < k ? expf(my_l - l0) : 0.f;
  float z = ex;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) z += __shfl_xor_sync(0xffffffffu, z, off);
  if (lane < k) {
    idx[t * k + lane] = my_e;
    gate[t * k + lane] = ex / z;
  }
}

cudaError_t launch_topk(const float* logits, const float* sel_bias, int64_t T, int E, int k,
                        int32_t* idx, float* gate, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  const int warps = 8;
  const unsigned grid = (unsigned)((T + warps - 1) / warps);
  const int vpl = (E + 31) / 32;
  switch (vpl) {
#define MOE_TOPK_CASE(N)                                                                    \
  case N:                                                                                   \
    return launch_pdl(topk_kernel<N>, dim3(grid), dim3(warps * 32), 0, s, logits, sel_bias, \
                      T, E, k, idx, gate);
    MOE_TOPK_CASE(1)
    MOE_TOPK_CASE(2)
    MOE_TOPK_CASE(3)
    MOE_TOPK_CASE(4)
    MOE_TOPK_CASE(5)
    MOE_TOPK_CASE(6)
    MOE_TOPK_CASE(7)
    MOE_TOPK_CASE(8)
#undef MOE_TOPK_CASE
    default:
      return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

// fp32 router on CUDA cores: logits[t,e] = sum_i x[t,i] W_r^T[e,i] + bias[e].
// One warp per token, experts in groups of 16: lane l accumulates, for each
// expert of the group, the products of the elements i = 4l .. 4l+3 of every
// 128-element chunk of d (chunks ascending), then a butterfly over the 32
// lanes sums the partials; lane j < 16 holds expert j's logit.  The x row is
// read through L1 once per expert group; W_r^T rows are read by every warp
// of the block from L1/L2.  The summation order is fixed, so the logits are
// identical on every run.
constexpr int kRouterWarps = 8;

__global__ void __launch_bounds__(32 * kRouterWarps)
    router_f32_kernel(const float* __restrict__ x, const float* __restrict__ wrT,
                      const float* __restrict__ bias, int64_t T, int d, int E,
                      float* __restrict__ logits) {
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t t = (int64_t)blockIdx.x * kRouterWarps + (threadIdx.x >> 5);
  if (t >= T) return;  // uniform per warp
  const float4* xr = reinterpret_cast<const float4*>(x + t * d);
  const int nch = d / 128;  // d % 64 == 0: the last chunk may be half
  const int tail = (d % 128) / 4;  // float4s in a half chunk (0 or 16)
  for (int e0 = 0; e0 < E; e0 += 16) {
    float acc[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) acc[j] = 0.f;
    for (int c = 0; c <= nch; ++c) {
      const int v = c * 32 + lane;  // float4 index in the row
      if (c == nch && lane >= tail) break;
      const float4 a = __ldg(xr + v);
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        if (e0 + j < E) {
          const float4 w = __ldg(reinterpret_cast<const float4*>(wrT + (int64_t)(e0 + j) * d) + v);
          acc[j] = fmaf(a.x, w.x, acc[j]);
          acc[j] = fmaf(a.y, w.y, acc[j]);
          acc[j] = fmaf(a.z, w.z, acc[j]);
          acc[j] = fmaf(a.w, w.w, acc[j]);
        }
      }
    }
#pragma unroll
    for (int j = 0; j < 16; ++j)
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) acc[j] += __shfl_xor_sync(0xffffffffu, acc[j], off);
    float mine = 0.f;
#pragma unroll
    for (int j = 0; j < 16; ++j)
      if (lane == j) mine = acc[j];
    const int e = e0 + lane;
    if (lane < 16 && e < E) logits[t * E + e] = bias ? mine + __ldg(bias + e) : mine;
  }
}

cudaError_t launch_router_f32(const float* x, const float* wrT, const float* bias, int64_t T,
                              int d, int E, float* logits, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  const unsigned grid = (unsigned)((T + kRouterWarps - 1) / kRouterWarps);
  return launch_pdl(router_f32_kernel, dim3(grid), dim3(32 * kRouterWarps), 0, s, x, wrT, bias,
                    T, d, E, logits);
}

}  // namespace moe
