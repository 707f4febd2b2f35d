// placement.cu - correlated expert placement ("Expert Coupling in MoE
// Pretraining", Abstract: place experts that are often selected together on
// the same GPU; Table III: the co-selection count W[e,e']; Table I caption:
// the placement is fit on other iterations than those it is evaluated on).
//
//  * co-selection counts on the GPU: W[e,e'] = number of ordered slot pairs
//    (a, b), a != b, of one token with idx[a] = e and idx[b] = e' (for a
//    routing of distinct experts: the tokens that select both e and e');
//  * the greedy fit on the host from those counts: each rank in turn is
//    seeded with the unassigned expert of largest row sum of W, then filled
//    with the unassigned expert of largest total co-selection with the
//    rank's members, until it holds E/ep experts (ties: lowest index).
#include <vector>

#include "kernels.cuh"

namespace moe {

namespace {

constexpr int kCoselThreads = 256;

// One token per thread.  With E <= 128 each block counts into an E x E
// histogram in shared memory and adds it to W once; larger E adds to W
// directly.  Integer sums, so the result does not depend on the order.
__global__ void __launch_bounds__(kCoselThreads)
    coselection_kernel(const int32_t* __restrict__ idx, int64_t T, int k, int E, int use_smem,
                       unsigned long long* __restrict__ W, Control* ctl) {
  extern __shared__ uint32_t hist[];
  pdl_wait();
  if (use_smem)
    for (int i = threadIdx.x; i < E * E; i += blockDim.x) hist[i] = 0;
  __syncthreads();
  bool bad = false;
  for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < T;
       t += (int64_t)gridDim.x * blockDim.x) {
    int e[16];
    bool tb = false;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      e[j] = j < k ? __ldg(idx + t * k + j) : 0;
      tb |= j < k && (e[j] < 0 || e[j] >= E);
    }
    bad |= tb;
    if (tb) continue;  // a token with an index outside [0, E) adds nothing
#pragma unroll
    for (int a = 0; a < 16; ++a)
#pragma unroll
      for (int b = 0; b < 16; ++b)
        if (a < k && b < k && a != b) {
          if (use_smem)
            atomicAdd(&hist[e[a] * E + e[b]], 1u);
          else
            atomicAdd(&W[e[a] * E + e[b]], 1ull);
        }
  }
  if (__syncthreads_or(bad) && threadIdx.x == 0) record_error(ctl, MOE_ERR_DEVICE_INDEX, 0xA00u);
  if (use_smem)
    for (int i = threadIdx.x; i < E * E; i += blockDim.x)
      if (hist[i]) atomicAdd(&W[i], (unsigned long long)hist[i]);
}

}  // namespace

cudaError_t launch_coselection(const int32_t* idx, int64_t T, int k, int E, uint64_t* W,
                               Control* ctl, cudaStream_t s) {
  cudaError_t e = cudaMemsetAsync(W, 0, sizeof(uint64_t) * E * E, s);
  if (e != cudaSuccess || T == 0) return e;
  const int use_smem = E <= 128 ? 1 : 0;
  const size_t smem = use_smem ? sizeof(uint32_t) * E * E : 0;
  if ((e = set_smem_limit((const void*)coselection_kernel, smem)) != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t need = (T + kCoselThreads - 1) / kCoselThreads;
  const unsigned grid = (unsigned)(need < 2 * sms ? need : 2 * sms);
  return launch_pdl(coselection_kernel, dim3(grid), dim3(kCoselThreads), smem, s, idx, T, k, E,
                    use_smem, reinterpret_cast<unsigned long long*>(W), ctl);
}

void fit_correlated_placement(const uint64_t* W, int E, int ep, int32_t* rank_of) {
  const int per = E / ep;
  std::vector<char> free_(E, 1);
  std::vector<uint64_t> rowsum(E, 0);
  for (int e = 0; e < E; ++e)
    for (int f = 0; f < E; ++f) rowsum[e] += W[(size_t)e * E + f];
  std::vector<uint64_t> gain(E);
  for (int r = 0; r < ep; ++r) {
    // seed: largest row sum, lowest index among equals
    int seed = -1;
    for (int e = 0; e < E; ++e)
      if (free_[e] && (seed < 0 || rowsum[e] > rowsum[seed])) seed = e;
    if (seed < 0) return;  // not reached: ep * (E/ep) == E experts to place
    free_[seed] = 0;
    rank_of[seed] = r;
    // co-selection of every free expert with the rank's members
    for (int e = 0; e < E; ++e) gain[e] = W[(size_t)e * E + seed];
    for (int n = 1; n < per; ++n) {
      int best = -1;
      for (int e = 0; e < E; ++e)
        if (free_[e] && (best < 0 || gain[e] > gain[best])) best = e;
      if (best < 0) return;
      free_[best] = 0;
      rank_of[best] = r;
      for (int e = 0; e < E; ++e) gain[e] += W[(size_t)e * E + best];
    }
  }
}

}  // namespace moe
