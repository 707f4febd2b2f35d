// kernels.cuh - launchers shared between the kernel files and the C ABI.
#pragma once

#include <mutex>
#include <vector>

#include "common.cuh"

namespace moe {

// Raise `kernel`'s dynamic shared-memory limit to at least `bytes` on the
// current device.  The limit belongs to each device's context, so it is
// recorded per (kernel, device); calls from several host threads are
// serialised.
inline cudaError_t set_smem_limit(const void* kernel, size_t bytes) {
  struct Done {
    const void* fn;
    int dev;
    size_t bytes;
  };
  static std::mutex mu;
  static std::vector<Done> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  Done* rec = nullptr;
  for (Done& d : done)
    if (d.fn == kernel && d.dev == dev) rec = &d;
  if (rec && rec->bytes >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e != cudaSuccess) return e;
  if (rec)
    rec->bytes = bytes;
  else
    done.push_back({kernel, dev, bytes});
  return cudaSuccess;
}

// Launch with programmatic stream serialization (see common.cuh).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t s, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// expert -> rank map passed by value to the layout kernels (E <= 256,
// ep <= 256, so a rank fits one byte)
struct RankMap {
  uint8_t r[256];
};

// ---- route.cu
// sel_bias [E] or NULL: added to the logits for the choice of experts only
cudaError_t launch_topk(const float* logits, const float* sel_bias, int64_t T, int E, int k,
                        int32_t* idx, float* gate, cudaStream_t s);
cudaError_t launch_router_f32(const float* x, const float* wrT, const float* bias, int64_t T,
                              int d, int E, float* logits, cudaStream_t s);

// ---- layout.cu
constexpr int kTokPerBlock = 128;        // tokens per lookback block (= one router tile)
constexpr int kLayoutThreads = 256;
constexpr int kMaxBins = 256 + 256 + 2;  // experts + ranks + two stat counters

inline int layout_blocks(int64_t T) { return (int)((T + kTokPerBlock - 1) / kTokPerBlock); }
inline int layout_bins(int E, int ep) { return E + (ep > 1 ? ep : 0) + 2; }
// Per-tile histogram counts are 16-bit (at most 128 tokens x k <= 16 per
// tile and bin).  Row stride (entries) of block_hist [bins][stride]: nb
// rounded up to a multiple of 8 so every row starts 16-byte aligned.
inline int layout_hist_stride(int nb) { return (nb + 7) & ~7; }

struct LayoutOut {
  int32_t *counts, *offsets, *row_token, *slot_row;
  int32_t *rank_counts, *rank_offsets, *send_token, *slot_send_row;
  moe_stats* stats;
};

// Scratch layout shared by every layout path: the control block, then
// kTotalsBytes for the per-bin totals, then the lookback status words
// [nb][bins] (zero between calls).
constexpr size_t kTotalsBytes = 4096;
static_assert(kTotalsBytes >= kMaxBins * sizeof(int32_t), "totals fit");

cudaError_t launch_layout(const int32_t* idx, int64_t T, int k, int E, int ep, const RankMap& map,
                          const LayoutOut& out, Control* ctl, uint64_t* status_words,
                          int32_t* totals, int stall_block, int64_t limit_ns, cudaStream_t s);
// the scatter half of the layout after the fused router, which left one
// histogram column per 128-token block in block_hist [bins][stride]
// (stride = layout_hist_stride(nb))
cudaError_t launch_layout_scatter(const int32_t* idx, int64_t T, int k, int E, int ep,
                                  const RankMap& map, const LayoutOut& out, Control* ctl,
                                  const uint16_t* block_hist, cudaStream_t s);

// ---- permute_combine.cu
// x_perm[r] = x[row_token[r]].  With slot_row non-NULL the copy runs in
// token order instead (x row t to rows slot_row[t*k + j]), same result.
cudaError_t launch_permute(const void* x, const int32_t* row_token, const int32_t* slot_row,
                           void* x_perm, int64_t T, int k, uint32_t row_bytes, cudaStream_t s);
cudaError_t launch_combine(int dtype, const void* y_perm, const int32_t* slot_row,
                           const float* gate, void* y, int64_t T, int d, int k, cudaStream_t s);

// ---- gemm_tc.cu (bf16, tcgen05)
// Grouped GEMM  out[r, :] = epilogue(A[r, :] . B_g^T)  for rows r of group g
// (rows [offsets[g], offsets[g+1])), with B_g rows [g*n_per_group, ...).
enum Epilogue { kEpiSwiGLU = 0, kEpiBF16 = 1 };
struct GemmArgs {
  const void* A;           // [rows, K] bf16 row-major
  int64_t rows;            // rows of A (tensor-map extent)
  const void* B;           // [G * n_per_group, K] bf16 row-major (K-major)
  const int32_t* offsets;  // [G+1] device, or NULL: one group of all `rows`
  int G;
  int K;
  int n_per_group;
  int n_out;               // valid output columns
  void* out;
  int64_t ld_out;          // output row stride in elements
  Control* ctl;
  // gather mode (gate/up GEMM only): A row r is row gather[r] of A, which
  // then has src_rows rows -- the permute fused into the operand load
  const int32_t* gather = nullptr;
  int64_t src_rows = 0;
  // combine fused into the epilogue (down GEMM on CTA pairs only): with y
  // set, the last of a token's k rows to be written for an N tile sums the
  // token's rows y[t] = sum_j gate[t,j] out[slot_row[t*k+j]] for that tile's
  // columns (fp32 in ascending j, one rounding: the combine kernel's
  // arithmetic).  arrive: T x (n_per_group / BN) counters, zero on entry.
  void* y = nullptr;
  const int32_t* row_token = nullptr;
  const int32_t* slot_row = nullptr;
  const float* gate = nullptr;
  int k = 0;
  int64_t T = 0;
  uint32_t* arrive = nullptr;
};
cudaError_t launch_gemm_tc(int epi, int bn, const GemmArgs& a, cudaStream_t s);
// ---- gemm_pair.cu: the same GEMM on CTA pairs (256-row tiles, tcgen05
// cta_group::2), bit-identical results; BN = 256, no gather
bool gemm_pair_supported(int epi, int bn, const GemmArgs& a);
cudaError_t launch_gemm_pair(int epi, int bn, const GemmArgs& a, cudaStream_t s);
bool make_kmajor_map(CUtensorMap* m, const void* base, int64_t rows, int K, int box_rows);
// 2-D fp32 [rows, cols] row-major, box of 32 columns (128 B) x box_rows,
// 128-byte swizzle (for tiled stores of swizzled shared-memory tiles)
bool make_f32_map(CUtensorMap* m, const void* base, int64_t rows, int cols, int box_rows);

// ---- route_tc.cu (bf16, tcgen05): router GEMM + bias + top-k + gates in one
// kernel, optionally with the layout histogram and its lookback scan
struct RouteArgs {
  const void* x;        // [T, d] bf16
  const void* wrT;      // [E16, d] bf16 (packed router)
  const float* bias;    // [E] or NULL
  const float* sel_bias = nullptr;  // [E] or NULL: added for the choice of experts only
  int64_t T;
  int d, E, k;
  float* logits;        // [T, E]
  int32_t* idx;         // [T, k]
  float* gate;          // [T, k]
  Control* ctl;
  // per-block dispatch histogram for the layout scatter (hist = false:
  // skipped): block_hist[bin][tile], layout_bins(E, ep) bins
  bool hist;
  int ep;
  RankMap map;
  uint16_t* block_hist;
};
cudaError_t launch_route_tc(const RouteArgs& a, cudaStream_t s);

// ---- ffn_fused.cu (bf16, tcgen05): gate/up GEMM + SwiGLU + down GEMM in
// one kernel for small f (H stays on chip); y_perm as moe_grouped_swiglu
struct FfnArgs {
  const void* A;             // gather: x [T, d]; else x_perm [rows, d]
  const int32_t* gather;     // row_token for gather mode, else NULL
  int64_t src_rows;          // T (gather mode)
  int64_t rows;              // T * k
  const int32_t* offsets;    // [E + 1]
  int G;                     // E
  int d, f;
  const void* wgu;           // packed [E * 2f, d] (gate rows then up rows per expert)
  const void* wdT;           // packed [E * d, f]
  void* y_perm;              // [rows, d]
  Control* ctl;
};
bool ffn_fused_supported(int d, int f);
cudaError_t launch_ffn_fused(const FfnArgs& a, cudaStream_t s);

// ---- gemm_simt.cu (fp32, CUDA cores)
// part 0: gate/up + SwiGLU into h; part 1: down into y_perm
cudaError_t launch_grouped_f32_part(int part, const float* x_perm, const int32_t* offsets, int E,
                                    int64_t R, int d, int f, int blk, const float* wgu,
                                    const float* wdT, float* h, float* y_perm, cudaStream_t s);

// ---- route_stats.cu
// Router statistics of a routing: margin [T] (double, may be NULL); counts[0]
// = T, and four counters added to counts[1..4] (zeroed by the caller):
// tokens with margin below `threshold`; against `recorded` (may be NULL) the
// tokens whose expert set changed, the experts swapped and the slots that
// differ.
cudaError_t launch_router_stats(const float* logits, const float* sel_bias, int64_t T, int E,
                                int k, const int32_t* idx, const int32_t* recorded,
                                double threshold, double* margin, unsigned long long* counts,
                                cudaStream_t s);
// Expert capacity: keep[a] = 1 for the first `cap` assignments of each
// expert in (choice rank, token) order, else 0; kept_gate[a] = gate[a] (1
// when gate is NULL) where kept, 0 where dropped (may be NULL).  Entries of
// out-of-range indices are not written (MOE_ERR_DEVICE_INDEX in ctl).
// H: capacity_scratch_bytes(T, k, E) of scratch (per-chunk counts).
size_t capacity_scratch_bytes(int64_t T, int k, int E);
cudaError_t launch_capacity_keep(const int32_t* idx, int64_t T, int k, int E, int64_t cap,
                                 const float* gate, int32_t* keep, float* kept_gate, int32_t* H,
                                 Control* ctl, cudaStream_t s);

// ---- placement.cu
// W[e * E + e'] = ordered slot pairs (a != b) of a token with experts
// (e, e') (zeroed here first); tokens with an index outside [0, E) add
// nothing and set MOE_ERR_DEVICE_INDEX.
cudaError_t launch_coselection(const int32_t* idx, int64_t T, int k, int E, uint64_t* W,
                               Control* ctl, cudaStream_t s);
// Greedy correlated placement from host counts W [E * E] (see placement.cu).
void fit_correlated_placement(const uint64_t* W, int E, int ep, int32_t* rank_of);

// ---- ep.cu (expert parallelism)
// expert -> owning rank and -> index among that rank's experts (ascending)
struct EpMaps {
  uint8_t rank[256];
  uint8_t local[256];
};
// where each destination rank's rows go when the pack stores them straight
// into the ranks' receive buffers (a kernel parameter: up to 256 ranks)
struct EpDest {
  void* recv_x;
  int32_t* recv_idx;
  float* recv_gate;
  int64_t row0;  // first row of this source's block there
  int64_t rows;  // rows of the block (send rows past it are not stored)
};
struct EpDests {
  EpDest d[256];
};
// where the return rows of each source rank go, and the received-row range
// of each source (base[s] .. base[s+1])
struct EpReturn {
  void* y_back;
  int64_t row0;
};
struct EpReturns {
  EpReturn d[256];
  int64_t base[257];
  int P;
};
// dests NULL: rows into send_x / send_idx / send_gate
cudaError_t launch_ep_pack(int dtype, const void* x, int64_t T, int d, int k, const int32_t* idx,
                           const float* gate, const int32_t* slot_send_row,
                           const int32_t* rank_offsets, int P, const EpMaps& maps, int E,
                           void* send_x, int32_t* send_idx, float* send_gate, int64_t cap,
                           const EpDests* dests, cudaStream_t s);
// every rank's flag array (P uint64 slots each), as this process maps them
struct EpFlags {
  uint64_t* flags[256];
};
cudaError_t launch_ep_signal_wait(const EpFlags& fl, int me, int P, uint64_t epoch,
                                  int64_t wait_ns, Control* ctl, cudaStream_t s);
// rets NULL: rows into y_ret
cudaError_t launch_ep_partial_combine(int dtype, const void* y_perm, const int32_t* slot_row,
                                      const int32_t* recv_idx, const float* recv_gate, int E_loc,
                                      void* y_ret, int64_t Tr, int d, int k, const EpReturns* rets,
                                      cudaStream_t s);
cudaError_t launch_ep_home_combine(int dtype, const void* y_back, const int32_t* slot_send_row,
                                   void* y, int64_t T, int d, int k, int64_t rows, cudaStream_t s);

// ---- pack.cu
// w_router NULL: only the experts; w_gate NULL: only the router
cudaError_t launch_pack(int dtype, int d, int E, int f, int blk, int E16, const void* w_router,
                        const void* w_gate, const void* w_up, const void* w_down, void* wrT,
                        void* wgu, void* wdT, cudaStream_t s);

}  // namespace moe
