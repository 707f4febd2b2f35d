// layout_static.cu - moe_dispatch_layout_static: the dispatch layout with its
// scratch memory in a fixed device array of this library, for callers that
// must not allocate device memory themselves.
//
// Who needs it: code that may not call cudaMalloc (or any allocator) on the
// path where it calls this library, for example an operator inside a host
// framework whose device memory was planned before it runs and which is
// handed only its inputs and outputs, or a C caller without a device
// allocator of its own.  cudaMalloc can also synchronise the whole device,
// which latency-sensitive callers avoid.  Such a caller cannot provide the
// workspace that moe_dispatch_layout takes, so this variant keeps the
// layout's scratch (control word, per-bin totals, decoupled-lookback status
// words) in `g_layout_scratch` below.
//
// The array is a file-scope __device__ variable: every GPU that loads the
// library holds its kStaticScratchBytes until the process exits.  Host code
// cannot pass the variable's name to a kernel (on the host it is only a
// stand-in, not a device address), so the first call on each device looks up
// its device address with cudaGetSymbolAddress while that device is current,
// and later calls reuse the address.
#include <mutex>

#include "checks.cuh"

namespace {

// the largest scratch this variant serves; larger shapes are rejected
constexpr size_t kStaticScratchBytes = size_t(1) << 20;
constexpr int kMaxDevices = 64;

__device__ __align__(256) uint8_t g_layout_scratch[kStaticScratchBytes];

std::mutex g_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

size_t round256(size_t x) { return (x + 255) / 256 * 256; }

// device address of g_layout_scratch on the current device (looked up once
// per device); NULL if the lookup failed
void* scratch_address() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_layout_scratch) != cudaSuccess) return nullptr;
    g_scratch_ptr[dev] = p;
  }
  return g_scratch_ptr[dev];
}

}  // namespace

extern "C" MOE_API moe_status moe_dispatch_layout_static(const moe_shape* s, const int32_t* topk_idx,
                                                         const int32_t* expert_rank_host,
                                                         const moe_layout* o, int32_t* device_status,
                                                         moe_stream_t stream) {
  using namespace moe;
  // the same checks, in the same order, as moe_dispatch_layout
  moe_status r = check_shape(s);
  if (r != MOE_OK) return r;
  if (!topk_idx && s->T > 0) return MOE_ERR_INVALID_ARG;
  if ((r = check_layout_ptrs(s, o)) != MOE_OK) return r;
  if (!aligned(topk_idx, 4) || (device_status && !aligned(device_status, 4))) return MOE_ERR_ALIGNMENT;

  // the scratch this shape needs, laid out as in moe_dispatch_layout
  const size_t nb = (size_t)layout_blocks(s->T), bins = (size_t)layout_bins(s->E, s->ep);
  const size_t off_totals = round256(sizeof(Control));
  const size_t off_status = off_totals + kTotalsBytes;
  const size_t need = off_status + round256(nb * bins * 8);
  if (need > kStaticScratchBytes) return MOE_ERR_WORKSPACE;

  RankMap map;
  if ((r = build_map(s, expert_rank_host, &map)) != MOE_OK) return r;

  uint8_t* base = static_cast<uint8_t*>(scratch_address());
  if (!base) return MOE_ERR_CUDA;
  cudaStream_t st = (cudaStream_t)stream;
  // The array keeps whatever the previous call left; the control word, the
  // ticket counter and the lookback status words must start at zero.
  if (cudaMemsetAsync(base, 0, need, st) != cudaSuccess) return MOE_ERR_CUDA;
  LayoutOut lo;
  lo.counts = o->expert_counts;
  lo.offsets = o->expert_offsets;
  lo.row_token = o->row_token;
  lo.slot_row = o->slot_row;
  lo.rank_counts = o->rank_counts;
  lo.rank_offsets = o->rank_offsets;
  lo.send_token = o->send_token;
  lo.slot_send_row = o->slot_send_row;
  lo.stats = o->stats;
  Control* ctl = reinterpret_cast<Control*>(base);
  if (launch_layout(topk_idx, s->T, s->k, s->E, s->ep, map, lo, ctl,
                    reinterpret_cast<uint64_t*>(base + off_status),
                    reinterpret_cast<int32_t*>(base + off_totals), -1, kWaitLimitNs, st) != cudaSuccess)
    return MOE_ERR_CUDA;
  // the device-side status of this call (MOE_OK, MOE_ERR_DEVICE_INDEX or
  // MOE_ERR_DEVICE_TIMEOUT), copied out for the caller
  if (device_status &&
      cudaMemcpyAsync(device_status, &ctl->status, sizeof(int32_t), cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}
