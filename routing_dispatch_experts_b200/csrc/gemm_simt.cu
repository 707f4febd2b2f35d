// gemm_simt.cu - grouped SwiGLU experts in fp32 on the CUDA cores.
//
// The fp32 workload keeps fp32 arithmetic end to end (tensor-core TF32 would
// round the inputs to 10-bit mantissas), so its grouped GEMMs are FMA
// kernels.  Each CTA computes a 64 x 64 output tile of one expert's rows with
// 256 threads (4 x 4 outputs each), staging 64 x 16 slices of the operands in
// shared memory; every output is one fmaf chain over k ascending, so results
// are deterministic.
//   gate/up:  h[r, n] = silu(sum_k x[r,k] Wg[e][k,n]) * (sum_k x[r,k] Wu[e][k,n])
//   down:     y[r, o] = sum_n h[r,n] Wd[e][n,o]
// ("Revisiting MoE and Dense Speed-Accuracy Comparisons", 2.1: SwiGLU).
// Operands come from the packed K-major weights: for gate/up, output column
// n of expert e is packed row (n / blk) * 2blk + n % blk (gate) and that
// plus blk (up) of a [2f, d] block; for down, row o of W_d^T [d, f].
#include <algorithm>

#include "kernels.cuh"

namespace moe {

namespace {

constexpr int TM = 64, TN = 64, TK = 16;

template <bool SWIGLU>
__global__ void __launch_bounds__(256) grouped_f32_kernel(const float* __restrict__ A,
                                                          const int32_t* __restrict__ offsets,
                                                          int E, int rows, int K, int N,
                                                          const float* __restrict__ W, int blk,
                                                          int64_t w_group_stride,
                                                          float* __restrict__ out) {
  __shared__ int tile_off[257];
  __shared__ int s_off[257];
  __shared__ float sA[TK][TM + 4];
  __shared__ float sG[TK][TN + 4];
  __shared__ float sU[SWIGLU ? TK : 1][TN + 4];
  const int tid = threadIdx.x;
  pdl_wait();
  // offsets clamped to [0, rows] and a negative group size read as empty: a
  // malformed offset array can never move a load or a store outside A / out
  for (int g = tid; g <= E; g += 256) s_off[g] = min(max(__ldg(offsets + g), 0), rows);
  __syncthreads();
  if (tid < 32) {
    int carry = 0;
    for (int g0 = 0; g0 < E; g0 += 32) {
      const int g = g0 + tid;
      const int v = g < E ? (max(s_off[g + 1] - s_off[g], 0) + TM - 1) / TM : 0;
      int incl = v;
      for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, incl, off);
        if (tid >= off) incl += o;
      }
      if (g < E) tile_off[g] = carry + incl - v;
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (tid == 0) tile_off[E] = carry;
  }
  __syncthreads();
  const int n_tiles = N / TN;
  const int total = tile_off[E] * n_tiles;
  for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
    const int mt = tile / n_tiles, nt = tile - mt * n_tiles;
    int lo = 1, hi = E;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (tile_off[mid] > mt) hi = mid; else lo = mid + 1;
    }
    const int e = lo - 1;
    const int row0 = s_off[e] + (mt - tile_off[e]) * TM;
    const int row_end = s_off[e + 1];
    const float* We = W + (int64_t)e * w_group_stride;
    const int tx = tid & 15, ty = tid >> 4;  // 16 x 16 threads, 4 x 4 outputs each
    float accg[4][4] = {}, accu[4][4] = {};
    for (int k0 = 0; k0 < K; k0 += TK) {
      // A slice: 64 rows x 16 k  (256 threads x 4 values)
      for (int i = tid; i < TM * TK; i += 256) {
        const int r = i / TK, kk = i % TK;
        const int row = row0 + r;
        sA[kk][r] = row < row_end ? __ldg(A + (int64_t)row * K + k0 + kk) : 0.f;
      }
      for (int i = tid; i < TN * TK; i += 256) {
        const int n = i / TK, kk = i % TK;
        const int col = nt * TN + n;
        int64_t wr;
        if (SWIGLU) wr = (int64_t)(col / blk) * 2 * blk + col % blk;
        else wr = col;
        sG[kk][n] = __ldg(We + wr * K + k0 + kk);
        if (SWIGLU) sU[kk][n] = __ldg(We + (wr + blk) * K + k0 + kk);
      }
      __syncthreads();
#pragma unroll
      for (int kk = 0; kk < TK; ++kk) {
        float a[4], g[4], u[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          a[i] = sA[kk][ty * 4 + i];
          g[i] = sG[kk][tx * 4 + i];
          if (SWIGLU) u[i] = sU[kk][tx * 4 + i];
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            accg[i][j] = fmaf(a[i], g[j], accg[i][j]);
            if (SWIGLU) accu[i][j] = fmaf(a[i], u[j], accu[i][j]);
          }
      }
      __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int row = row0 + ty * 4 + i;
      if (row >= row_end) continue;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int col = nt * TN + tx * 4 + j;
        float v = accg[i][j];
        if (SWIGLU) v = v / (1.f + expf(-v)) * accu[i][j];
        out[(int64_t)row * N + col] = v;
      }
    }
  }
}

}  // namespace

cudaError_t launch_grouped_f32_part(int part, const float* x_perm, const int32_t* offsets, int E,
                                    int64_t R, int d, int f, int blk, const float* wgu,
                                    const float* wdT, float* h, float* y_perm, cudaStream_t s) {
  if (R == 0) return cudaSuccess;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t mt_max = (R + TM - 1) / TM + E;
  if (part == 0) {
    const int grid1 = (int)std::min<int64_t>(mt_max * (f / TN), (int64_t)sms * 8);
    return launch_pdl(grouped_f32_kernel<true>, dim3(grid1), dim3(256), 0, s, x_perm, offsets, E,
                      (int)R, d, f, wgu, blk, (int64_t)2 * f * d, h);
  } else {
    const int grid2 = (int)std::min<int64_t>(mt_max * (d / TN), (int64_t)sms * 8);
    return launch_pdl(grouped_f32_kernel<false>, dim3(grid2), dim3(256), 0, s,
                      static_cast<const float*>(h), offsets, E, (int)R, f, d, wdT, blk,
                      (int64_t)d * f, y_perm);
  }
}

}  // namespace moe
