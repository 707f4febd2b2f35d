// pack.cu - one-time rearrangement of the layer's weights into the kernels'
// K-major operand layout.
//
// The pages store the router as "ME" = [d, E] and the expert FFNs as
// "EMH" = [E, d, f] (gate, up) and "EHM" = [E, f, d] (down) ("Revisiting
// MoE and Dense Speed-Accuracy Comparisons", Table 1).  The tensor-core
// kernels read every operand K-major (the reduction index contiguous), so
// each matrix is transposed once, through 32 x 32 shared-memory tiles:
//   W_r   [d, E]    -> [E16, d]         (rows E..E16-1 zero)
//   W_g/u [E, d, f] -> [E, 2f, d]       (per block of blk columns: blk gate
//                                        rows, then the same blk up rows)
//   W_d   [E, f, d] -> [E, d, f]
#include "kernels.cuh"

namespace moe {

namespace {

// dst[b][map(c)][r] = src[b][r][c] for a batch of [rows, cols] matrices;
// map(c) = (c / blk) * blk_stride + blk_off + c % blk.
template <typename T>
__global__ void __launch_bounds__(256) transpose_kernel(const T* __restrict__ src, T* __restrict__ dst,
                                                        int rows, int cols, int64_t src_bstride,
                                                        int64_t dst_bstride, int blk, int blk_stride,
                                                        int blk_off) {
  __shared__ T tile[32][33];
  const int b = blockIdx.z;
  const int r0 = blockIdx.y * 32, c0 = blockIdx.x * 32;
  const T* s = src + (int64_t)b * src_bstride;
  T* d = dst + (int64_t)b * dst_bstride;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // 32 x 8
  for (int i = ty; i < 32; i += 8) {
    const int r = r0 + i, c = c0 + tx;
    if (r < rows && c < cols) tile[i][tx] = s[(int64_t)r * cols + c];
  }
  __syncthreads();
  for (int i = ty; i < 32; i += 8) {
    const int c = c0 + i, r = r0 + tx;
    if (r < rows && c < cols) {
      const int64_t drow = (int64_t)(c / blk) * blk_stride + blk_off + c % blk;
      d[drow * rows + r] = tile[tx][i];
    }
  }
}

template <typename T>
cudaError_t transpose(const void* src, void* dst, int batch, int rows, int cols, int64_t sbs,
                      int64_t dbs, int blk, int blk_stride, int blk_off, cudaStream_t s) {
  dim3 grid((cols + 31) / 32, (rows + 31) / 32, batch);
  transpose_kernel<T><<<grid, 256, 0, s>>>(static_cast<const T*>(src), static_cast<T*>(dst), rows,
                                           cols, sbs, dbs, blk, blk_stride, blk_off);
  return cudaGetLastError();
}

template <typename T>
cudaError_t pack_all(int d, int E, int f, int blk, int E16, const void* w_router,
                     const void* w_gate, const void* w_up, const void* w_down, void* wrT, void* wgu,
                     void* wdT, cudaStream_t s) {
  cudaError_t err = cudaSuccess;
  if (w_router) {
    err = cudaMemsetAsync(wrT, 0, sizeof(T) * (size_t)E16 * d, s);
    if (err != cudaSuccess) return err;
    // router [d, E] -> [E, d]
    err = transpose<T>(w_router, wrT, 1, d, E, 0, 0, E, 0, 0, s);
    if (err != cudaSuccess) return err;
  }
  if (!w_gate) return cudaSuccess;  // the router alone
  // gate / up [E][d, f] -> [E][2f, d], blocks of blk rows interleaved
  const int64_t gu_stride = (int64_t)2 * f * d;
  err = transpose<T>(w_gate, wgu, E, d, f, (int64_t)d * f, gu_stride, blk, 2 * blk, 0, s);
  if (err != cudaSuccess) return err;
  err = transpose<T>(w_up, wgu, E, d, f, (int64_t)d * f, gu_stride, blk, 2 * blk, blk, s);
  if (err != cudaSuccess) return err;
  // down [E][f, d] -> [E][d, f]
  return transpose<T>(w_down, wdT, E, f, d, (int64_t)f * d, (int64_t)d * f, d, 0, 0, s);
}

}  // namespace

cudaError_t launch_pack(int dtype, int d, int E, int f, int blk, int E16, const void* w_router,
                        const void* w_gate, const void* w_up, const void* w_down, void* wrT,
                        void* wgu, void* wdT, cudaStream_t s) {
  if (dtype == MOE_BF16)
    return pack_all<uint16_t>(d, E, f, blk, E16, w_router, w_gate, w_up, w_down, wrT, wgu, wdT, s);
  return pack_all<float>(d, E, f, blk, E16, w_router, w_gate, w_up, w_down, wrT, wgu, wdT, s);
}

}  // namespace moe
