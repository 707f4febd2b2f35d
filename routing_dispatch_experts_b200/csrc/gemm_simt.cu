// gemm_simt.cu - grouped SwiGLU experts in fp32 on the CUDA cores.
//
// The fp32 workload keeps fp32 arithmetic end to end (tensor-core TF32 would
// round the inputs to 10-bit mantissas), so its grouped GEMMs are FMA
// kernels.  Each CTA computes a 128 x 64 output tile of one expert's rows
// with 256 threads (8 rows x 4 columns each, two 16-byte shared-memory loads
// of A and one of each weight per k), staging 16-wide k slices of the
// operands in shared memory, double-buffered: the next slice is loaded into
// registers while the current one is multiplied.  Every output is one fmaf
// chain over k ascending, so results are deterministic.
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

constexpr int TM = 128, TN = 64, TK = 16;
constexpr int PAD = 4;  // keeps rows 16-byte aligned, spreads the transposed stores

template <bool SWIGLU>
__global__ void __launch_bounds__(256, 2) grouped_f32_kernel(const float* __restrict__ A,
                                                             const int32_t* __restrict__ offsets,
                                                             int E, int rows, int K, int N,
                                                             const float* __restrict__ W, int blk,
                                                             int64_t w_group_stride,
                                                             float* __restrict__ out) {
  __shared__ int tile_off[257];
  __shared__ int s_off[257];
  __shared__ __align__(16) float sA[2][TK][TM + PAD];
  __shared__ __align__(16) float sG[2][TK][TN + PAD];
  __shared__ __align__(16) float sU[SWIGLU ? 2 : 1][SWIGLU ? TK : 1][TN + PAD];
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
  const int tx = tid & 15, ty = tid >> 4;  // columns 4 tx .. +3, rows 8 ty .. +7
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
    // this thread's global loads of a k slice: two float4 of A (rows
    // idx >> 2, k quad idx & 3, idx = tid and tid + 256) and one of each
    // weight (column tid >> 2, k quad tid & 3)
    const int bn = tid >> 2, bq = tid & 3;
    const int col = nt * TN + bn;
    const int64_t wr = SWIGLU ? (int64_t)(col / blk) * 2 * blk + col % blk : col;
    float4 ra[2], rg, ru;
    auto load = [&](int k0) {
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int idx = tid + 256 * j;
        const int row = row0 + (idx >> 2);
        ra[j] = row < row_end ? __ldg(reinterpret_cast<const float4*>(A + (int64_t)row * K + k0) + (idx & 3))
                              : make_float4(0.f, 0.f, 0.f, 0.f);
      }
      rg = __ldg(reinterpret_cast<const float4*>(We + wr * K + k0) + bq);
      if (SWIGLU) ru = __ldg(reinterpret_cast<const float4*>(We + (wr + blk) * K + k0) + bq);
    };
    auto store = [&](int buf) {
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int idx = tid + 256 * j;
        const int r = idx >> 2, q = idx & 3;
        sA[buf][4 * q + 0][r] = ra[j].x;
        sA[buf][4 * q + 1][r] = ra[j].y;
        sA[buf][4 * q + 2][r] = ra[j].z;
        sA[buf][4 * q + 3][r] = ra[j].w;
      }
      sG[buf][4 * bq + 0][bn] = rg.x;
      sG[buf][4 * bq + 1][bn] = rg.y;
      sG[buf][4 * bq + 2][bn] = rg.z;
      sG[buf][4 * bq + 3][bn] = rg.w;
      if (SWIGLU) {
        sU[buf][4 * bq + 0][bn] = ru.x;
        sU[buf][4 * bq + 1][bn] = ru.y;
        sU[buf][4 * bq + 2][bn] = ru.z;
        sU[buf][4 * bq + 3][bn] = ru.w;
      }
    };
    float accg[8][4] = {}, accu[SWIGLU ? 8 : 1][4] = {};
    load(0);
    store(0);
    __syncthreads();
    int buf = 0;
    for (int k0 = 0; k0 < K; k0 += TK) {
      const bool more = k0 + TK < K;
      if (more) load(k0 + TK);
#pragma unroll
      for (int kk = 0; kk < TK; ++kk) {
        const float4 a0 = *reinterpret_cast<const float4*>(&sA[buf][kk][ty * 8]);
        const float4 a1 = *reinterpret_cast<const float4*>(&sA[buf][kk][ty * 8 + 4]);
        const float4 g4 = *reinterpret_cast<const float4*>(&sG[buf][kk][tx * 4]);
        const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
        const float g[4] = {g4.x, g4.y, g4.z, g4.w};
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) accg[i][j] = fmaf(a[i], g[j], accg[i][j]);
        if (SWIGLU) {
          const float4 u4 = *reinterpret_cast<const float4*>(&sU[buf][kk][tx * 4]);
          const float u[4] = {u4.x, u4.y, u4.z, u4.w};
#pragma unroll
          for (int i = 0; i < 8; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) accu[SWIGLU ? i : 0][j] = fmaf(a[i], u[j], accu[SWIGLU ? i : 0][j]);
        }
      }
      if (more) {
        store(buf ^ 1);
        __syncthreads();
        buf ^= 1;
      }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int row = row0 + ty * 8 + i;
      if (row >= row_end) continue;
      float v[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        v[j] = accg[i][j];
        if (SWIGLU) v[j] = v[j] / (1.f + expf(-v[j])) * accu[SWIGLU ? i : 0][j];
      }
      *reinterpret_cast<float4*>(out + (int64_t)row * N + nt * TN + tx * 4) =
          make_float4(v[0], v[1], v[2], v[3]);
    }
    __syncthreads();  // every thread is done with the buffers before the next tile
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
