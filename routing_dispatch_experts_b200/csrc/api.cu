// api.cu - the C ABI: argument checks, workspace carving, kernel sequencing.
//
// Host code only; every step of the layer runs in the kernels of the other
// files.  Nothing here allocates device memory or synchronises a stream
// (except moe_get_device_status, whose job is to read the device status).
#include <algorithm>
#include <cmath>
#include <cstring>

#include "checks.cuh"

using namespace moe;

namespace {

constexpr size_t kAlign = 256;

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

int gu_block(int f) { return f % 128 == 0 ? 128 : 64; }

int pad16(int E) { return (E + 15) / 16 * 16; }

// ---- scratch workspace: control block, per-bin totals, lookback words
struct Scratch {
  Control* ctl;
  int32_t* totals;
  uint64_t* status;      // lookback words, zero between calls
  uint16_t* block_hist;  // per-block histogram rows of the fused router (16-bit counts)
};

// the lookback status words of the layout; the same bytes hold the
// per-chunk counts of moe_capacity_keep
size_t status_bytes(const moe_shape* s) {
  const size_t nb = (size_t)layout_blocks(s->T), bins = (size_t)layout_bins(s->E, s->ep);
  return align_up(std::max(nb * bins * 8, capacity_scratch_bytes(s->T, s->k, s->E)));
}

size_t scratch_bytes(const moe_shape* s) {
  const size_t nb = (size_t)layout_blocks(s->T), bins = (size_t)layout_bins(s->E, s->ep);
  const size_t hs = (size_t)layout_hist_stride((int)nb);
  return align_up(sizeof(Control)) + kTotalsBytes + status_bytes(s) + align_up(hs * bins * 2);
}

Scratch carve_scratch(const moe_shape* s, void* ws) {
  uint8_t* p = static_cast<uint8_t*>(ws);
  Scratch sc;
  sc.ctl = reinterpret_cast<Control*>(p);
  p += align_up(sizeof(Control));
  sc.totals = reinterpret_cast<int32_t*>(p);
  p += kTotalsBytes;
  sc.status = reinterpret_cast<uint64_t*>(p);
  p += status_bytes(s);
  sc.block_hist = reinterpret_cast<uint16_t*>(p);
  return sc;
}

// ---- packed weights
struct Packed {
  const void* wrT;
  const void* wgu;
  const void* wdT;
};

size_t packed_bytes(const moe_shape* s) {
  const size_t es = esize(s->dtype);
  return align_up((size_t)pad16(s->E) * s->d * es) + align_up((size_t)s->E * 2 * s->f * s->d * es) +
         align_up((size_t)s->E * s->d * s->f * es);
}

Packed carve_packed(const moe_shape* s, const void* packed) {
  const size_t es = esize(s->dtype);
  const uint8_t* p = static_cast<const uint8_t*>(packed);
  Packed pk;
  pk.wrT = p;
  p += align_up((size_t)pad16(s->E) * s->d * es);
  pk.wgu = p;
  p += align_up((size_t)s->E * 2 * s->f * s->d * es);
  pk.wdT = p;
  return pk;
}

// ---- forward intermediates placed after the scratch
struct FwdBufs {
  float* logits;
  int32_t* idx;
  float* gate;
  moe_layout lay;
  void* x_perm;
  void* h;
  void* y_perm;
  uint32_t* arrive;
};

// arrival counters of the combine fused into the down GEMM: one per token
// and 64-column block of d (enough for any N tile width)
size_t arrive_count(const moe_shape* s) { return (size_t)s->T * (size_t)((s->d + 63) / 64); }

size_t forward_bytes(const moe_shape* s) {
  const size_t R = (size_t)s->T * s->k, es = esize(s->dtype);
  size_t n = scratch_bytes(s);
  n += align_up((size_t)s->T * s->E * 4);      // logits
  n += 2 * align_up(R * 4);                     // idx, gate
  n += align_up((size_t)s->E * 4) + align_up((size_t)(s->E + 1) * 4);
  n += 2 * align_up(R * 4);                     // row_token, slot_row
  n += align_up((size_t)s->ep * 4) + align_up((size_t)(s->ep + 1) * 4);
  n += 2 * align_up(R * 4);                     // send_token, slot_send_row
  n += align_up(sizeof(moe_stats));
  n += align_up(R * s->d * es) + align_up(R * s->f * es) + align_up(R * s->d * es);
  n += align_up(arrive_count(s) * 4);           // fused-combine arrival counters
  return n;
}

FwdBufs carve_forward(const moe_shape* s, void* ws, const moe_forward_buffers* b) {
  const size_t R = (size_t)s->T * s->k, es = esize(s->dtype);
  uint8_t* p = static_cast<uint8_t*>(ws) + scratch_bytes(s);
  auto take = [&p](size_t bytes) {
    void* q = p;
    p += align_up(bytes);
    return q;
  };
  FwdBufs f;
  f.logits = static_cast<float*>(take((size_t)s->T * s->E * 4));
  f.idx = static_cast<int32_t*>(take(R * 4));
  f.gate = static_cast<float*>(take(R * 4));
  f.lay.expert_counts = static_cast<int32_t*>(take((size_t)s->E * 4));
  f.lay.expert_offsets = static_cast<int32_t*>(take((size_t)(s->E + 1) * 4));
  f.lay.row_token = static_cast<int32_t*>(take(R * 4));
  f.lay.slot_row = static_cast<int32_t*>(take(R * 4));
  f.lay.rank_counts = static_cast<int32_t*>(take((size_t)s->ep * 4));
  f.lay.rank_offsets = static_cast<int32_t*>(take((size_t)(s->ep + 1) * 4));
  f.lay.send_token = static_cast<int32_t*>(take(R * 4));
  f.lay.slot_send_row = static_cast<int32_t*>(take(R * 4));
  f.lay.stats = static_cast<moe_stats*>(take(sizeof(moe_stats)));
  f.x_perm = take(R * s->d * es);
  f.h = take(R * s->f * es);
  f.y_perm = take(R * s->d * es);
  f.arrive = static_cast<uint32_t*>(take(arrive_count(s) * 4));
  if (b) {
    if (b->logits) f.logits = b->logits;
    if (b->topk_idx) f.idx = b->topk_idx;
    if (b->topk_gate) f.gate = b->topk_gate;
    if (b->layout.expert_counts) f.lay.expert_counts = b->layout.expert_counts;
    if (b->layout.expert_offsets) f.lay.expert_offsets = b->layout.expert_offsets;
    if (b->layout.row_token) f.lay.row_token = b->layout.row_token;
    if (b->layout.slot_row) f.lay.slot_row = b->layout.slot_row;
    if (b->layout.rank_counts) f.lay.rank_counts = b->layout.rank_counts;
    if (b->layout.rank_offsets) f.lay.rank_offsets = b->layout.rank_offsets;
    if (b->layout.send_token) f.lay.send_token = b->layout.send_token;
    if (b->layout.slot_send_row) f.lay.slot_send_row = b->layout.slot_send_row;
    if (b->layout.stats) f.lay.stats = b->layout.stats;
    if (b->x_perm) f.x_perm = b->x_perm;
    if (b->h) f.h = b->h;
    if (b->y_perm) f.y_perm = b->y_perm;
  }
  return f;
}

moe_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

// ---- the steps, after their arguments are checked
moe_status do_route(const moe_shape* s, const void* x, const Packed* pk, const float* bias,
                    const float* sel_bias, float* logits, int32_t* idx, float* gate, Control* ctl,
                    cudaStream_t st) {
  if (x) {
    cudaError_t e;
    if (s->dtype == MOE_BF16) {
      // router GEMM, top-k and gates in one tcgen05 kernel
      RouteArgs a{};
      a.x = x;
      a.wrT = pk->wrT;
      a.bias = bias;
      a.sel_bias = sel_bias;
      a.T = s->T;
      a.d = s->d;
      a.E = s->E;
      a.k = s->k;
      a.logits = logits;
      a.idx = idx;
      a.gate = gate;
      a.ctl = ctl;
      a.hist = false;
      a.ep = s->ep;
      return cuda_status(launch_route_tc(a, st));
    } else {
      e = launch_router_f32(static_cast<const float*>(x), static_cast<const float*>(pk->wrT), bias,
                            s->T, s->d, s->E, logits, st);
    }
    if (e != cudaSuccess) return MOE_ERR_CUDA;
  }
  return cuda_status(launch_topk(logits, sel_bias, s->T, s->E, s->k, idx, gate, st));
}

moe_status do_layout(const moe_shape* s, const int32_t* idx, const RankMap& map,
                     const moe_layout* o, const Scratch& sc, int stall, int64_t limit,
                     cudaStream_t st) {
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
  return cuda_status(launch_layout(idx, s->T, s->k, s->E, s->ep, map, lo, sc.ctl, sc.status,
                                   sc.totals, stall, limit, st));
}

// gate/up GEMM + SwiGLU (part 0) or down GEMM (part 1).  With `gather`
// (bf16 only) the gate/up GEMM reads its rows straight from x through the
// permutation instead of from x_perm.
// Which tensor-core GEMM engine runs a grouped GEMM: one CTA per 128-row
// tile (gemm_tc.cu) or CTA pairs on 256-row tiles (gemm_pair.cu).
enum Engine {
  kEngineAuto = 0,       // the library's choice (below)
  kEngineSingle = 1,     // one CTA per tile for both GEMMs
  kEnginePair = 2,       // CTA pairs for both GEMMs where they apply
  kEnginePairDown = 3,   // CTA pairs for the down GEMM only
  kEnginePairGateUp = 4  // CTA pairs for the gate/up GEMM only
};

// The library's choice, from full-size measurements on B200 (flushed
// forwards): CTA pairs pay for the down GEMM once its K loop has 16 or more
// k-blocks (f = 1536: -10% per clock, its staged epilogue leaving the
// one-CTA ring three stages deep; f = 1024: the top-2 and top-6 forwards 1-2%
// faster), not for the gate/up GEMM (more DRAM re-reads of its operands:
// 9.06 vs 7.0 GB per large-workload launch); the pair's TMA gather4 row
// gather issues 32 row loads per stage and measured twice as slow as the
// one-CTA cp.async gather.
bool pair_chosen(int epi, const GemmArgs& a) {
  return epi == kEpiBF16 && a.gather == nullptr && a.K >= 16 * 64;
}

// The combine can be summed in the down GEMM's epilogue when the library
// runs that GEMM on CTA pairs with 256-column tiles (bf16).
bool combine_fusable(const moe_shape* s) {
  if (s->dtype != MOE_BF16 || s->d % 256 != 0 || s->f <= 512) return false;
  GemmArgs a{};
  a.K = s->f;
  a.n_per_group = s->d;
  return pair_chosen(kEpiBF16, a) && gemm_pair_supported(kEpiBF16, 256, a);
}

cudaError_t launch_gemm(int epi, int bn, const GemmArgs& a, int engine, cudaStream_t st) {
  bool pair = false;
  switch (engine) {
    case kEnginePair: pair = true; break;
    case kEnginePairDown: pair = epi == kEpiBF16; break;
    case kEnginePairGateUp: pair = epi == kEpiSwiGLU; break;
    case kEngineAuto: pair = pair_chosen(epi, a); break;
    default: break;
  }
  if (pair && gemm_pair_supported(epi, bn, a)) return launch_gemm_pair(epi, bn, a, st);
  return launch_gemm_tc(epi, bn, a, st);
}

// The combine fused into the down GEMM (CTA pairs only; see GemmArgs).
struct FusedCombine {
  void* y = nullptr;
  const int32_t* row_token = nullptr;
  const int32_t* slot_row = nullptr;
  const float* gate = nullptr;
  uint32_t* arrive = nullptr;
};

moe_status do_grouped_part(int part, const moe_shape* s, const void* a_rows,
                           const int32_t* gather, const int32_t* offsets, const Packed* pk,
                           void* h, void* y_perm, Control* ctl, cudaStream_t st,
                           int engine = kEngineAuto, const FusedCombine* fc = nullptr) {
  const int64_t R = s->T * (int64_t)s->k;
  if (s->dtype == MOE_F32)
    return cuda_status(launch_grouped_f32_part(part, static_cast<const float*>(a_rows), offsets,
                                               s->E, R, s->d, s->f, gu_block(s->f),
                                               static_cast<const float*>(pk->wgu),
                                               static_cast<const float*>(pk->wdT),
                                               static_cast<float*>(h), static_cast<float*>(y_perm),
                                               st));
  GemmArgs a{};
  a.offsets = offsets;
  a.G = s->E;
  a.rows = R;
  a.ctl = ctl;
  if (part == 0) {
    a.A = a_rows;
    a.gather = gather;
    a.src_rows = s->T;
    a.B = pk->wgu;
    a.K = s->d;
    a.n_per_group = 2 * s->f;
    a.n_out = s->f;
    a.out = h;
    a.ld_out = s->f;
    return cuda_status(launch_gemm(kEpiSwiGLU, 2 * gu_block(s->f), a, engine, st));
  }
  a.A = h;
  a.B = pk->wdT;
  a.K = s->f;
  a.n_per_group = s->d;
  a.n_out = s->d;
  a.out = y_perm;
  a.ld_out = s->d;
  // short K (f <= 512): 128-column tiles, so two CTAs fit per SM
  const int bn = (s->d % 256 == 0 && s->f > 512) ? 256 : (s->d % 128 == 0 ? 128 : 64);
  if (fc) {
    a.y = fc->y;
    a.row_token = fc->row_token;
    a.slot_row = fc->slot_row;
    a.gate = fc->gate;
    a.k = s->k;
    a.T = s->T;
    a.arrive = fc->arrive;
  }
  return cuda_status(launch_gemm(kEpiBF16, bn, a, engine, st));
}

moe_status do_grouped(const moe_shape* s, const void* x_perm, const int32_t* offsets,
                      const Packed* pk, void* h, void* y_perm, Control* ctl, cudaStream_t st,
                      int engine = kEngineAuto) {
  moe_status r = do_grouped_part(0, s, x_perm, nullptr, offsets, pk, h, y_perm, ctl, st, engine);
  if (r != MOE_OK) return r;
  return do_grouped_part(1, s, x_perm, nullptr, offsets, pk, h, y_perm, ctl, st, engine);
}

moe_status layout_entry(const moe_shape* s, const int32_t* idx, const int32_t* host_map,
                        const moe_layout* o, void* ws, size_t ws_bytes, int stall, int64_t limit,
                        cudaStream_t st) {
  moe_status r = check_shape(s);
  if (r != MOE_OK) return r;
  if ((!idx && s->T > 0) || !ws) return MOE_ERR_INVALID_ARG;
  if ((r = check_layout_ptrs(s, o)) != MOE_OK) return r;
  if (!aligned(idx, 4) || !aligned(ws, kAlign)) return MOE_ERR_ALIGNMENT;
  if (ws_bytes < scratch_bytes(s)) return MOE_ERR_WORKSPACE;
  RankMap map;
  if ((r = build_map(s, host_map, &map)) != MOE_OK) return r;
  return do_layout(s, idx, map, o, carve_scratch(s, ws), stall, limit, st);
}

// The gathered gate/up GEMM reads each row of x once per expert that picks
// it, 128 bytes at a time; that pays while x stays in the 126 MB L2, and a
// separate streaming permute wins once x is much larger (measured on B200:
// faster at x = 8 and 67 MB, slower at 268 MB).
constexpr int64_t kGatherMaxBytes = 96ll << 20;
bool gather_fits(const moe_shape* s) {
  return s->dtype == MOE_BF16 && s->T * (int64_t)s->d * 2 <= kGatherMaxBytes;
}

// The forward; with `routed` the caller's (r_idx, r_gate) replace the router
// (no logits, no router kernel) and the standalone dispatch layout runs.
moe_status forward_impl(const moe_shape* s, const void* x, const void* packed, const float* bias,
                        const int32_t* expert_rank_host, void* y, const moe_forward_buffers* buffers,
                        void* ws, size_t ws_bytes, cudaStream_t st, cudaEvent_t* ev,
                        bool routed = false, const int32_t* r_idx = nullptr,
                        const float* r_gate = nullptr, const float* sel_bias = nullptr,
                        int options = 0) {
  moe_status r = check_shape(s);
  if (r != MOE_OK) return r;
  if (!ws) return MOE_ERR_INVALID_ARG;
  if (!aligned(ws, kAlign)) return MOE_ERR_ALIGNMENT;
  if (ws_bytes < forward_bytes(s)) return MOE_ERR_WORKSPACE;
  RankMap map;
  if ((r = build_map(s, expert_rank_host, &map)) != MOE_OK) return r;
  if (s->T == 0) return MOE_OK;
  if (!x || !packed || !y || (routed && !r_idx)) return MOE_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(y, 16) || !aligned(packed, kAlign) || (bias && !aligned(bias, 4)) ||
      (sel_bias && !aligned(sel_bias, 4)))
    return MOE_ERR_ALIGNMENT;
  if (routed && (!aligned(r_idx, 4) || (r_gate && !aligned(r_gate, 4)))) return MOE_ERR_ALIGNMENT;
  FwdBufs f = carve_forward(s, ws, buffers);
  if ((r = check_layout_ptrs(s, &f.lay)) != MOE_OK) return r;
  if (!aligned(f.logits, 4) || !aligned(f.idx, 4) || !aligned(f.gate, 4) || !aligned(f.x_perm, 16) ||
      !aligned(f.h, 16) || !aligned(f.y_perm, 16))
    return MOE_ERR_ALIGNMENT;
  const Scratch sc = carve_scratch(s, ws);
  const Packed pk = carve_packed(s, packed);
  // stage markers for moe_forward_timed: 0 route, 1 layout, 2 permute,
  // 3 gate/up GEMM, 4 down GEMM, 5 combine, 6 end
  auto mark = [&](int i) { return ev ? cuda_status(cudaEventRecord(ev[i], st)) : MOE_OK; };
  LayoutOut lo;
  lo.counts = f.lay.expert_counts;
  lo.offsets = f.lay.expert_offsets;
  lo.row_token = f.lay.row_token;
  lo.slot_row = f.lay.slot_row;
  lo.rank_counts = f.lay.rank_counts;
  lo.rank_offsets = f.lay.rank_offsets;
  lo.send_token = f.lay.send_token;
  lo.slot_send_row = f.lay.slot_send_row;
  lo.stats = f.lay.stats;
  const bool bf16 = s->dtype == MOE_BF16;
  // small f: the whole expert FFN and the combine in one kernel
  const bool fused = bf16 && ffn_fused_supported(s->d, s->f);
  if ((r = mark(0)) != MOE_OK) return r;
  // routing and dispatch layout
  if (routed) {
    if ((r = mark(1)) != MOE_OK) return r;
    if ((r = do_layout(s, r_idx, map, &f.lay, sc, -1, kWaitLimitNs, st)) != MOE_OK) return r;
    if ((r = mark(2)) != MOE_OK) return r;
  } else if (bf16) {
    // router + top-k + gates + per-tile dispatch histogram in one kernel
    RouteArgs a{};
    a.x = x;
    a.wrT = pk.wrT;
    a.bias = bias;
    a.sel_bias = sel_bias;
    a.T = s->T;
    a.d = s->d;
    a.E = s->E;
    a.k = s->k;
    a.logits = f.logits;
    a.idx = f.idx;
    a.gate = f.gate;
    a.ctl = sc.ctl;
    a.hist = true;
    a.ep = s->ep;
    a.map = map;
    a.block_hist = sc.block_hist;
    if ((r = cuda_status(launch_route_tc(a, st))) != MOE_OK) return r;
    if ((r = mark(1)) != MOE_OK) return r;
    // the scatter half of the layout
    if ((r = cuda_status(launch_layout_scatter(f.idx, s->T, s->k, s->E, s->ep, map, lo, sc.ctl,
                                               sc.block_hist, st))) != MOE_OK)
      return r;
    if ((r = mark(2)) != MOE_OK) return r;
  } else {
    if ((r = do_route(s, x, &pk, bias, sel_bias, f.logits, f.idx, f.gate, sc.ctl, st)) != MOE_OK)
      return r;
    if ((r = mark(1)) != MOE_OK) return r;
    if ((r = do_layout(s, f.idx, map, &f.lay, sc, -1, kWaitLimitNs, st)) != MOE_OK) return r;
    if ((r = mark(2)) != MOE_OK) return r;
  }
  // expert FFN
  if (bf16) {
    if (fused) {
      FfnArgs fa{};
      const bool g = gather_fits(s);
      if (!g && (r = cuda_status(launch_permute(x, f.lay.row_token, f.lay.slot_row, f.x_perm, s->T,
                                                s->k, (uint32_t)(s->d * 2), st))) != MOE_OK)
        return r;
      if ((r = mark(3)) != MOE_OK) return r;
      fa.A = g ? x : f.x_perm;
      fa.gather = g ? f.lay.row_token : nullptr;
      fa.src_rows = s->T;
      fa.rows = s->T * (int64_t)s->k;
      fa.offsets = f.lay.expert_offsets;
      fa.G = s->E;
      fa.d = s->d;
      fa.f = s->f;
      fa.wgu = pk.wgu;
      fa.wdT = pk.wdT;
      fa.y_perm = f.y_perm;
      fa.ctl = sc.ctl;
      if ((r = cuda_status(launch_ffn_fused(fa, st))) != MOE_OK) return r;
      if ((r = mark(4)) != MOE_OK) return r;
    } else if (gather_fits(s)) {
      // the permute is fused into the gate/up GEMM's operand loads
      if ((r = mark(3)) != MOE_OK) return r;
      if ((r = do_grouped_part(0, s, x, f.lay.row_token, f.lay.expert_offsets, &pk, f.h, f.y_perm,
                               sc.ctl, st)) != MOE_OK)
        return r;
    } else {
      // x larger than L2: copy in token order, reading each row of x once
      if ((r = cuda_status(launch_permute(x, f.lay.row_token, f.lay.slot_row, f.x_perm, s->T,
                                          s->k, (uint32_t)(s->d * esize(s->dtype)), st))) != MOE_OK)
        return r;
      if ((r = mark(3)) != MOE_OK) return r;
      if ((r = do_grouped_part(0, s, f.x_perm, nullptr, f.lay.expert_offsets, &pk, f.h, f.y_perm,
                               sc.ctl, st)) != MOE_OK)
        return r;
    }
  } else {
    if ((r = cuda_status(launch_permute(x, f.lay.row_token, nullptr, f.x_perm, s->T, s->k,
                                        (uint32_t)(s->d * esize(s->dtype)), st))) != MOE_OK)
      return r;
    if ((r = mark(3)) != MOE_OK) return r;
    if ((r = do_grouped_part(0, s, f.x_perm, nullptr, f.lay.expert_offsets, &pk, f.h, f.y_perm,
                             sc.ctl, st)) != MOE_OK)
      return r;
  }
  // on request, the combine in the down GEMM's epilogue where that GEMM
  // runs on pairs (measured slower than the separate combine kernel on the
  // large workload, so not the default)
  const bool fuse_combine = (options & MOE_FWD_COMBINE_IN_DOWN) && !fused && combine_fusable(s);
  if (!fused) {
    if ((r = mark(4)) != MOE_OK) return r;
    FusedCombine fc;
    if (fuse_combine) {
      fc.y = y;
      fc.row_token = f.lay.row_token;
      fc.slot_row = f.lay.slot_row;
      fc.gate = routed ? r_gate : f.gate;
      fc.arrive = f.arrive;
      if ((r = cuda_status(cudaMemsetAsync(f.arrive, 0, arrive_count(s) * 4, st))) != MOE_OK)
        return r;
    }
    if ((r = do_grouped_part(1, s, nullptr, nullptr, f.lay.expert_offsets, &pk, f.h, f.y_perm,
                             sc.ctl, st, kEngineAuto, fuse_combine ? &fc : nullptr)) != MOE_OK)
      return r;
  }
  if ((r = mark(5)) != MOE_OK) return r;
  if (!fuse_combine &&
      (r = cuda_status(launch_combine(s->dtype, f.y_perm, f.lay.slot_row, routed ? r_gate : f.gate,
                                      y, s->T, s->d, s->k, st))) != MOE_OK)
    return r;
  return mark(6);
}

// ---- expert parallelism: the receiving rank's workspace
// Received rows are routed over E_loc = E/ep local experts plus one group
// (index E_loc) that collects the slots whose expert another rank holds.
struct EpRecv {
  Scratch sc;
  LayoutOut lo;
  void* x_perm;
  void* h;
  void* y_perm;
};

size_t ep_recv_bytes(const moe_shape* s) {
  const int El = s->E / s->ep + 1;
  const size_t R = (size_t)s->T * s->k, es = esize(s->dtype);
  const size_t nb = (size_t)layout_blocks(s->T), bins = (size_t)layout_bins(El, 1);
  size_t n = align_up(sizeof(Control)) + kTotalsBytes + align_up(nb * bins * 8);
  n += align_up((size_t)El * 4) + align_up((size_t)(El + 1) * 4) + 2 * align_up(R * 4);
  n += align_up(R * s->d * es) + align_up(R * s->f * es) + align_up(R * s->d * es);
  return n;
}

EpRecv carve_ep_recv(const moe_shape* s, void* ws) {
  const int El = s->E / s->ep + 1;
  const size_t R = (size_t)s->T * s->k, es = esize(s->dtype);
  const size_t nb = (size_t)layout_blocks(s->T), bins = (size_t)layout_bins(El, 1);
  uint8_t* p = static_cast<uint8_t*>(ws);
  auto take = [&p](size_t bytes) {
    void* q = p;
    p += align_up(bytes);
    return q;
  };
  EpRecv r{};
  r.sc.ctl = static_cast<Control*>(take(sizeof(Control)));
  r.sc.totals = static_cast<int32_t*>(static_cast<void*>(p));
  p += kTotalsBytes;
  r.sc.status = static_cast<uint64_t*>(take(nb * bins * 8));
  r.sc.block_hist = nullptr;
  r.lo.counts = static_cast<int32_t*>(take((size_t)El * 4));
  r.lo.offsets = static_cast<int32_t*>(take((size_t)(El + 1) * 4));
  r.lo.row_token = static_cast<int32_t*>(take(R * 4));
  r.lo.slot_row = static_cast<int32_t*>(take(R * 4));
  r.lo.rank_counts = r.lo.rank_offsets = r.lo.send_token = r.lo.slot_send_row = nullptr;
  r.lo.stats = nullptr;
  r.x_perm = take(R * s->d * es);
  r.h = take(R * s->f * es);
  r.y_perm = take(R * s->d * es);
  return r;
}

moe_status route_impl(const moe_shape* s, const void* x, const void* packed, const float* bias,
                      const float* sel_bias, float* logits, int32_t* topk_idx, float* topk_gate,
                      void* ws, size_t ws_bytes, cudaStream_t st) {
  moe_status r = check_shape(s);
  if (r != MOE_OK) return r;
  if (s->T > 0 && (!logits || !topk_idx || !topk_gate)) return MOE_ERR_INVALID_ARG;
  if (x && (!packed || !ws)) return MOE_ERR_INVALID_ARG;
  if ((x && !aligned(x, 16)) || (packed && !aligned(packed, kAlign)) || !aligned(logits, 4) ||
      !aligned(topk_idx, 4) || !aligned(topk_gate, 4) || (bias && !aligned(bias, 4)) ||
      (sel_bias && !aligned(sel_bias, 4)) || (ws && !aligned(ws, kAlign)))
    return MOE_ERR_ALIGNMENT;
  if (ws && ws_bytes < scratch_bytes(s)) return MOE_ERR_WORKSPACE;
  if (s->T == 0) return MOE_OK;
  Packed pk{};
  if (packed) pk = carve_packed(s, packed);
  Control* ctl = ws ? carve_scratch(s, ws).ctl : nullptr;
  return do_route(s, x, &pk, bias, sel_bias, logits, topk_idx, topk_gate, ctl, st);
}

moe_status gather_impl(const moe_shape* s, const void* x, const int32_t* row_token,
                       const int32_t* offsets, const void* packed, void* h, void* y_perm, void* ws,
                       size_t ws_bytes, int engine, cudaStream_t st) {
  moe_status r = check_shape(s);
  if (r != MOE_OK) return r;
  if (s->dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
  if (s->T == 0) return MOE_OK;
  if (!x || !row_token || !offsets || !packed || !h || !y_perm || !ws) return MOE_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(h, 16) || !aligned(y_perm, 16) || !aligned(offsets, 4) ||
      !aligned(row_token, 4) || !aligned(packed, kAlign) || !aligned(ws, kAlign))
    return MOE_ERR_ALIGNMENT;
  if (ws_bytes < scratch_bytes(s)) return MOE_ERR_WORKSPACE;
  const Packed pk = carve_packed(s, packed);
  Control* ctl = carve_scratch(s, ws).ctl;
  if ((r = do_grouped_part(0, s, x, row_token, offsets, &pk, h, y_perm, ctl, st, engine)) != MOE_OK)
    return r;
  return do_grouped_part(1, s, x, nullptr, offsets, &pk, h, y_perm, ctl, st, engine);
}

}  // namespace

extern "C" {

const char* moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
    case MOE_ERR_ALIGNMENT: return "MOE_ERR_ALIGNMENT";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
    case MOE_ERR_DEVICE_TIMEOUT: return "MOE_ERR_DEVICE_TIMEOUT";
    case MOE_ERR_DEVICE_INDEX: return "MOE_ERR_DEVICE_INDEX";
  }
  return "MOE_ERR_UNKNOWN";
}

moe_status moe_scratch_size(const moe_shape* s, size_t* bytes) {
  moe_status r = check_shape(s);
  if (r != MOE_OK) return r;
  if (!bytes) return MOE_ERR_INVALID_ARG;
  *bytes = scratch_bytes(s);
  return MOE_OK;
}

moe_status moe_forward_workspace_size(const moe_shape* s, size_t* bytes) {
  moe_status r = check_shape(s);
  if (r != MOE_OK) return r;
  if (!bytes) return MOE_ERR_INVALID_ARG;
  *bytes = forward_bytes(s);
  return MOE_OK;
}

moe_status moe_workspace_init(void* ws, size_t bytes, moe_stream_t stream) {
  if (!ws) return MOE_ERR_INVALID_ARG;
  return cuda_status(cudaMemsetAsync(ws, 0, bytes, (cudaStream_t)stream));
}

moe_status moe_packed_weights_size(const moe_shape* s, size_t* bytes) {
  moe_status r = check_shape(s);
  if (r != MOE_OK) return r;
  if (!bytes) return MOE_ERR_INVALID_ARG;
  *bytes = packed_bytes(s);
  return MOE_OK;
}

moe_status moe_pack_weights(const moe_shape* s, const void* w_router, const void* w_gate,
                            const void* w_up, const void* w_down, void* packed,
                            size_t packed_bytes_, moe_stream_t stream) {
  moe_status r = check_shape(s);
  if (r != MOE_OK) return r;
  // the router alone (no expert weights), the experts alone (no router), or both
  const bool experts = w_gate || w_up || w_down;
  if (experts && (!w_gate || !w_up || !w_down)) return MOE_ERR_INVALID_ARG;
  if ((!w_router && !experts) || !packed) return MOE_ERR_INVALID_ARG;
  const size_t es = esize(s->dtype);
  for (const void* p : {w_router, w_gate, w_up, w_down})
    if (p && !aligned(p, es)) return MOE_ERR_ALIGNMENT;
  if (!aligned(packed, kAlign)) return MOE_ERR_ALIGNMENT;
  if (packed_bytes_ < packed_bytes(s)) return MOE_ERR_WORKSPACE;
  Packed pk = carve_packed(s, packed);
  return cuda_status(launch_pack(s->dtype, s->d, s->E, s->f, gu_block(s->f), pad16(s->E), w_router,
                                 w_gate, w_up, w_down, const_cast<void*>(pk.wrT),
                                 const_cast<void*>(pk.wgu), const_cast<void*>(pk.wdT),
                                 (cudaStream_t)stream));
}

moe_status moe_unpacked_workspace_size(const moe_shape* s, size_t* bytes) {
  moe_status r = check_shape(s);
  if (r != MOE_OK) return r;
  if (!bytes) return MOE_ERR_INVALID_ARG;
  *bytes = scratch_bytes(s) + packed_bytes(s);
  return MOE_OK;
}

moe_status moe_route_unpacked(const moe_shape* s, const void* x, const void* w_router,
                              const float* bias, float* logits, int32_t* topk_idx,
                              float* topk_gate, void* ws, size_t ws_bytes, moe_stream_t stream) {
  moe_status r = check_shape(s);
  if (r != MOE_OK) return r;
  if (!x || !w_router || !ws) return MOE_ERR_INVALID_ARG;
  if (!aligned(w_router, esize(s->dtype)) || !aligned(ws, kAlign)) return MOE_ERR_ALIGNMENT;
  if (ws_bytes < scratch_bytes(s) + packed_bytes(s)) return MOE_ERR_WORKSPACE;
  if (s->T == 0) return MOE_OK;
  // the router block of a packed buffer, built in the workspace after the
  // scratch, then the packed path
  void* packed = static_cast<uint8_t*>(ws) + scratch_bytes(s);
  const Packed pk = carve_packed(s, packed);
  cudaStream_t st = (cudaStream_t)stream;
  if ((r = cuda_status(launch_pack(s->dtype, s->d, s->E, s->f, gu_block(s->f), pad16(s->E),
                                   w_router, nullptr, nullptr, nullptr, const_cast<void*>(pk.wrT),
                                   nullptr, nullptr, st))) != MOE_OK)
    return r;
  return route_impl(s, x, packed, bias, nullptr, logits, topk_idx, topk_gate, ws,
                    scratch_bytes(s), st);
}

moe_status moe_grouped_swiglu_unpacked(const moe_shape* s, const void* x_perm,
                                       const int32_t* offsets, const void* w_gate,
                                       const void* w_up, const void* w_down, void* h,
                                       void* y_perm, void* ws, size_t ws_bytes,
                                       moe_stream_t stream) {
  moe_status r = check_shape(s);
  if (r != MOE_OK) return r;
  if (!w_gate || !w_up || !w_down || !ws) return MOE_ERR_INVALID_ARG;
  const int es = esize(s->dtype);
  if (!aligned(w_gate, es) || !aligned(w_up, es) || !aligned(w_down, es) || !aligned(ws, kAlign))
    return MOE_ERR_ALIGNMENT;
  if (ws_bytes < scratch_bytes(s) + packed_bytes(s)) return MOE_ERR_WORKSPACE;
  if (s->T == 0) return MOE_OK;
  void* packed = static_cast<uint8_t*>(ws) + scratch_bytes(s);
  const Packed pk = carve_packed(s, packed);
  cudaStream_t st = (cudaStream_t)stream;
  if ((r = cuda_status(launch_pack(s->dtype, s->d, s->E, s->f, gu_block(s->f), pad16(s->E),
                                   nullptr, w_gate, w_up, w_down, nullptr,
                                   const_cast<void*>(pk.wgu), const_cast<void*>(pk.wdT), st))) !=
      MOE_OK)
    return r;
  return moe_grouped_swiglu(s, x_perm, offsets, packed, h, y_perm, ws, scratch_bytes(s), stream);
}

moe_status moe_route(const moe_shape* s, const void* x, const void* packed, const float* bias,
                     float* logits, int32_t* topk_idx, float* topk_gate, void* ws,
                     size_t ws_bytes, moe_stream_t stream) {
  return route_impl(s, x, packed, bias, nullptr, logits, topk_idx, topk_gate, ws, ws_bytes,
                    (cudaStream_t)stream);
}

moe_status moe_route_selection_bias(const moe_shape* s, const void* x, const void* packed,
                                    const float* bias, const float* selection_bias, float* logits,
                                    int32_t* topk_idx, float* topk_gate, void* ws, size_t ws_bytes,
                                    moe_stream_t stream) {
  if (!selection_bias) return MOE_ERR_INVALID_ARG;
  return route_impl(s, x, packed, bias, selection_bias, logits, topk_idx, topk_gate, ws, ws_bytes,
                    (cudaStream_t)stream);
}

moe_status moe_router_stats(const moe_shape* s, const float* logits, const float* selection_bias,
                            const int32_t* topk_idx, const int32_t* recorded_idx, double threshold,
                            double* margin, moe_router_counts* stats, moe_stream_t stream) {
  moe_status r = check_shape(s);
  if (r != MOE_OK) return r;
  if (!stats || (s->T > 0 && !logits) || (recorded_idx && !topk_idx)) return MOE_ERR_INVALID_ARG;
  if (!(threshold >= 0.0)) return MOE_ERR_INVALID_ARG;
  if (!aligned(stats, 8) || (logits && !aligned(logits, 4)) || (margin && !aligned(margin, 8)) ||
      (selection_bias && !aligned(selection_bias, 4)) || (topk_idx && !aligned(topk_idx, 4)) ||
      (recorded_idx && !aligned(recorded_idx, 4)))
    return MOE_ERR_ALIGNMENT;
  cudaStream_t st = (cudaStream_t)stream;
  // the kernel writes the token count and adds to the other counters
  static_assert(sizeof(moe_router_counts) == 5 * sizeof(unsigned long long), "five counters");
  if (cudaMemsetAsync(stats, 0, sizeof(moe_router_counts), st) != cudaSuccess) return MOE_ERR_CUDA;
  return cuda_status(launch_router_stats(logits, selection_bias, s->T, s->E, s->k, topk_idx,
                                         recorded_idx, threshold, margin,
                                         reinterpret_cast<unsigned long long*>(stats), st));
}

moe_status moe_capacity_keep(const moe_shape* s, const int32_t* topk_idx, const float* topk_gate,
                             double capacity_factor, int32_t* keep, float* kept_gate,
                             int64_t* capacity, void* ws, size_t ws_bytes, moe_stream_t stream) {
  moe_status r = check_shape(s);
  if (r != MOE_OK) return r;
  if (!(capacity_factor > 0.0) || !(capacity_factor < 1e9) || !ws) return MOE_ERR_INVALID_ARG;
  // the factor times an expert's mean load, rounded up
  const int64_t cap = (int64_t)std::ceil(capacity_factor * (double)s->T * s->k / s->E);
  if (capacity) *capacity = cap;
  if (s->T == 0) return MOE_OK;
  if (!topk_idx || !keep) return MOE_ERR_INVALID_ARG;
  if (!aligned(topk_idx, 4) || !aligned(keep, 4) || (topk_gate && !aligned(topk_gate, 4)) ||
      (kept_gate && !aligned(kept_gate, 4)) || !aligned(ws, kAlign))
    return MOE_ERR_ALIGNMENT;
  if (ws_bytes < scratch_bytes(s)) return MOE_ERR_WORKSPACE;
  cudaStream_t st = (cudaStream_t)stream;
  const size_t R = (size_t)s->T * s->k;
  // entries with an out-of-range expert are written by no block: they read 0
  if (cudaMemsetAsync(keep, 0, R * 4, st) != cudaSuccess) return MOE_ERR_CUDA;
  if (kept_gate && cudaMemsetAsync(kept_gate, 0, R * 4, st) != cudaSuccess) return MOE_ERR_CUDA;
  // the per-chunk counts borrow the layout's lookback words, which must be
  // zero again before the next layout on this workspace
  const Scratch sc = carve_scratch(s, ws);
  if ((r = cuda_status(launch_capacity_keep(topk_idx, s->T, s->k, s->E, cap, topk_gate, keep,
                                            kept_gate, reinterpret_cast<int32_t*>(sc.status),
                                            sc.ctl, st))) != MOE_OK)
    return r;
  return cuda_status(
      cudaMemsetAsync(sc.status, 0, capacity_scratch_bytes(s->T, s->k, s->E), st));
}

moe_status moe_coselection_counts(const moe_shape* s, const int32_t* topk_idx, uint64_t* counts,
                                  void* ws, size_t ws_bytes, moe_stream_t stream) {
  moe_status r = check_shape(s);
  if (r != MOE_OK) return r;
  if (!counts || !ws || (s->T > 0 && !topk_idx)) return MOE_ERR_INVALID_ARG;
  if (!aligned(counts, 8) || (topk_idx && !aligned(topk_idx, 4)) || !aligned(ws, kAlign))
    return MOE_ERR_ALIGNMENT;
  if (ws_bytes < scratch_bytes(s)) return MOE_ERR_WORKSPACE;
  return cuda_status(launch_coselection(topk_idx, s->T, s->k, s->E, counts,
                                        carve_scratch(s, ws).ctl, (cudaStream_t)stream));
}

moe_status moe_fit_placement(int32_t E, int32_t ep, const uint64_t* counts_host,
                             int32_t* expert_rank_host) {
  if (E < 1 || E > 256 || ep < 1 || ep > E || E % ep != 0 || !counts_host || !expert_rank_host)
    return MOE_ERR_INVALID_ARG;
  fit_correlated_placement(counts_host, E, ep, expert_rank_host);
  return MOE_OK;
}

moe_status moe_ep_pack(const moe_shape* s, const void* x, const int32_t* topk_idx,
                       const float* topk_gate, const int32_t* expert_rank_host,
                       const moe_layout* layout, void* send_x, int32_t* send_idx,
                       float* send_gate, int64_t send_rows, moe_stream_t stream) {
  moe_status r = check_shape(s);
  if (r != MOE_OK) return r;
  if (s->ep < 2) return MOE_ERR_INVALID_ARG;
  if (send_rows < 0) return MOE_ERR_INVALID_ARG;
  if (s->T == 0 || send_rows == 0) return MOE_OK;
  if (!x || !topk_idx || !layout || !layout->slot_send_row || !layout->rank_offsets || !send_x ||
      !send_idx || !send_gate)
    return MOE_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(send_x, 16) || !aligned(topk_idx, 4) ||
      !aligned(layout->slot_send_row, 4) || !aligned(layout->rank_offsets, 4) ||
      !aligned(send_idx, 4) || !aligned(send_gate, 4) || (topk_gate && !aligned(topk_gate, 4)))
    return MOE_ERR_ALIGNMENT;
  RankMap map;
  if ((r = build_map(s, expert_rank_host, &map)) != MOE_OK) return r;
  EpMaps m{};
  int next[256] = {0};
  for (int e = 0; e < s->E; ++e) {
    m.rank[e] = map.r[e];
    m.local[e] = (uint8_t)next[map.r[e]]++;
  }
  return cuda_status(launch_ep_pack(s->dtype, x, s->T, s->d, s->k, topk_idx, topk_gate,
                                    layout->slot_send_row, layout->rank_offsets, s->ep, m, s->E,
                                    send_x, send_idx, send_gate, send_rows, nullptr,
                                    (cudaStream_t)stream));
}

moe_status moe_ep_dispatch_peer(const moe_shape* s, const void* x, const int32_t* topk_idx,
                                const float* topk_gate, const int32_t* expert_rank_host,
                                const moe_layout* layout, const moe_ep_peer_dest* dests_host,
                                moe_stream_t stream) {
  moe_status r = check_shape(s);
  if (r != MOE_OK) return r;
  if (s->ep < 2 || !dests_host) return MOE_ERR_INVALID_ARG;
  EpDests dd{};
  int64_t cap = 0;
  for (int q = 0; q < s->ep; ++q) {
    const moe_ep_peer_dest& d = dests_host[q];
    if (d.rows < 0 || d.row0 < 0) return MOE_ERR_INVALID_ARG;
    if (d.rows > 0) {
      if (!d.recv_x || !d.recv_idx || !d.recv_gate) return MOE_ERR_INVALID_ARG;
      if (!aligned(d.recv_x, 16) || !aligned(d.recv_idx, 4) || !aligned(d.recv_gate, 4))
        return MOE_ERR_ALIGNMENT;
    }
    dd.d[q].recv_x = d.recv_x;
    dd.d[q].recv_idx = d.recv_idx;
    dd.d[q].recv_gate = d.recv_gate;
    dd.d[q].row0 = d.row0;
    dd.d[q].rows = d.rows;
    cap += d.rows;
  }
  if (s->T == 0 || cap == 0) return MOE_OK;
  if (!x || !topk_idx || !layout || !layout->slot_send_row || !layout->rank_offsets)
    return MOE_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(topk_idx, 4) || !aligned(layout->slot_send_row, 4) ||
      !aligned(layout->rank_offsets, 4) || (topk_gate && !aligned(topk_gate, 4)))
    return MOE_ERR_ALIGNMENT;
  RankMap map;
  if ((r = build_map(s, expert_rank_host, &map)) != MOE_OK) return r;
  EpMaps m{};
  int next[256] = {0};
  for (int e = 0; e < s->E; ++e) {
    m.rank[e] = map.r[e];
    m.local[e] = (uint8_t)next[map.r[e]]++;
  }
  return cuda_status(launch_ep_pack(s->dtype, x, s->T, s->d, s->k, topk_idx, topk_gate,
                                    layout->slot_send_row, layout->rank_offsets, s->ep, m, s->E,
                                    nullptr, nullptr, nullptr, cap, &dd, (cudaStream_t)stream));
}

moe_status moe_ep_expert_workspace_size(const moe_shape* s, size_t* bytes) {
  moe_status r = check_shape(s);
  if (r != MOE_OK) return r;
  if (!bytes || s->ep < 2) return MOE_ERR_INVALID_ARG;
  *bytes = ep_recv_bytes(s);
  return MOE_OK;
}

// the receiving rank's experts; the return rows go to y_ret, or with
// `rets` straight to their source ranks' buffers
static moe_status ep_expert_impl(const moe_shape* s, const void* recv_x, const int32_t* recv_idx,
                          const float* recv_gate, const void* packed_local, void* y_ret,
                          const EpReturns* rets, void* ws, size_t ws_bytes, cudaStream_t st) {
  moe_status r = check_shape(s);
  if (r != MOE_OK) return r;
  if (s->ep < 2 || !ws) return MOE_ERR_INVALID_ARG;
  if (!aligned(ws, kAlign)) return MOE_ERR_ALIGNMENT;
  if (ws_bytes < ep_recv_bytes(s)) return MOE_ERR_WORKSPACE;
  if (s->T == 0) return MOE_OK;
  if (!recv_x || !recv_idx || !recv_gate || !packed_local || (!y_ret && !rets))
    return MOE_ERR_INVALID_ARG;
  if (!aligned(recv_x, 16) || (y_ret && !aligned(y_ret, 16)) || !aligned(recv_idx, 4) ||
      !aligned(recv_gate, 4) || !aligned(packed_local, kAlign))
    return MOE_ERR_ALIGNMENT;
  const int El = s->E / s->ep;
  const EpRecv rv = carve_ep_recv(s, ws);
  // the local experts' packed weights: a packed buffer of E/ep experts
  moe_shape loc = *s;
  loc.E = El;
  loc.ep = 1;
  loc.k = std::min(s->k, El);  // only E, d, f and dtype shape the packed buffer
  const Packed pk = carve_packed(&loc, packed_local);
  // layout of the received rows over the local experts plus the
  // "held elsewhere" group El (no rank dispatch: ep = 1)
  RankMap one;
  std::memset(&one, 0, sizeof(one));
  if ((r = cuda_status(launch_layout(recv_idx, s->T, s->k, El + 1, 1, one, rv.lo, rv.sc.ctl,
                                     rv.sc.status, rv.sc.totals, -1, kWaitLimitNs, st))) != MOE_OK)
    return r;
  // expert FFN over groups 0..El-1: their rows are [offsets[0], offsets[El])
  const int64_t R = s->T * (int64_t)s->k;
  if (s->dtype == MOE_BF16 && ffn_fused_supported(s->d, s->f)) {
    FfnArgs fa{};
    fa.A = recv_x;
    fa.gather = rv.lo.row_token;
    fa.src_rows = s->T;
    fa.rows = R;
    fa.offsets = rv.lo.offsets;
    fa.G = El;
    fa.d = s->d;
    fa.f = s->f;
    fa.wgu = pk.wgu;
    fa.wdT = pk.wdT;
    fa.y_perm = rv.y_perm;
    fa.ctl = rv.sc.ctl;
    if ((r = cuda_status(launch_ffn_fused(fa, st))) != MOE_OK) return r;
  } else {
    loc.T = s->T;
    loc.k = s->k;
    const bool g = s->dtype == MOE_BF16;
    if (!g && (r = cuda_status(launch_permute(recv_x, rv.lo.row_token, nullptr, rv.x_perm, s->T,
                                              s->k, (uint32_t)(s->d * esize(s->dtype)), st))) !=
                  MOE_OK)
      return r;
    if ((r = do_grouped_part(0, &loc, g ? recv_x : rv.x_perm, g ? rv.lo.row_token : nullptr,
                             rv.lo.offsets, &pk, rv.h, rv.y_perm, rv.sc.ctl, st)) != MOE_OK)
      return r;
    if ((r = do_grouped_part(1, &loc, nullptr, nullptr, rv.lo.offsets, &pk, rv.h, rv.y_perm,
                             rv.sc.ctl, st)) != MOE_OK)
      return r;
  }
  return cuda_status(launch_ep_partial_combine(s->dtype, rv.y_perm, rv.lo.slot_row, recv_idx,
                                               recv_gate, El, y_ret, s->T, s->d, s->k, rets, st));
}

moe_status moe_ep_expert_forward(const moe_shape* s, const void* recv_x, const int32_t* recv_idx,
                                 const float* recv_gate, const void* packed_local, void* y_ret,
                                 void* ws, size_t ws_bytes, moe_stream_t stream) {
  if (s && s->T > 0 && !y_ret) return MOE_ERR_INVALID_ARG;
  return ep_expert_impl(s, recv_x, recv_idx, recv_gate, packed_local, y_ret, nullptr, ws,
                        ws_bytes, (cudaStream_t)stream);
}

moe_status moe_ep_expert_forward_peer(const moe_shape* s, const void* recv_x,
                                      const int32_t* recv_idx, const float* recv_gate,
                                      const void* packed_local, const moe_ep_peer_return* rets_host,
                                      void* ws, size_t ws_bytes, moe_stream_t stream) {
  moe_status r = check_shape(s);
  if (r != MOE_OK) return r;
  if (s->ep < 2 || !rets_host) return MOE_ERR_INVALID_ARG;
  EpReturns rr{};
  rr.P = s->ep;
  int64_t base = 0;
  for (int q = 0; q < s->ep; ++q) {
    const moe_ep_peer_return& b = rets_host[q];
    if (b.rows < 0 || b.row0 < 0) return MOE_ERR_INVALID_ARG;
    if (b.rows > 0 && !b.y_back) return MOE_ERR_INVALID_ARG;
    if (b.rows > 0 && !aligned(b.y_back, 16)) return MOE_ERR_ALIGNMENT;
    rr.d[q].y_back = b.y_back;
    rr.d[q].row0 = b.row0;
    rr.base[q] = base;
    base += b.rows;
  }
  rr.base[s->ep] = base;
  if (base != s->T) return MOE_ERR_INVALID_ARG;  // the blocks tile the received rows
  return ep_expert_impl(s, recv_x, recv_idx, recv_gate, packed_local, nullptr, &rr, ws, ws_bytes,
                        (cudaStream_t)stream);
}

static moe_status ep_signal_impl(uint64_t* const* flags_host, int32_t rank, int32_t P, uint64_t epoch,
                          void* ws, int64_t wait_ns, cudaStream_t st) {
  if (P < 1 || P > 256 || rank < 0 || rank >= P || !flags_host || !ws || epoch == 0)
    return MOE_ERR_INVALID_ARG;
  if (!aligned(ws, kAlign)) return MOE_ERR_ALIGNMENT;
  EpFlags fl{};
  for (int q = 0; q < P; ++q) {
    if (!flags_host[q]) return MOE_ERR_INVALID_ARG;
    if (!aligned(flags_host[q], 8)) return MOE_ERR_ALIGNMENT;
    fl.flags[q] = flags_host[q];
  }
  return cuda_status(
      launch_ep_signal_wait(fl, rank, P, epoch, wait_ns, static_cast<Control*>(ws), st));
}

moe_status moe_ep_signal_wait(uint64_t* const* flags_host, int32_t rank, int32_t P,
                              uint64_t epoch, void* ws, moe_stream_t stream) {
  return ep_signal_impl(flags_host, rank, P, epoch, ws, kWaitLimitNs, (cudaStream_t)stream);
}

moe_status moe_debug_ep_signal_wait(uint64_t* const* flags_host, int32_t rank, int32_t P,
                                    uint64_t epoch, void* ws, int64_t wait_limit_ns,
                                    moe_stream_t stream) {
  if (wait_limit_ns <= 0 || wait_limit_ns > kWaitLimitNs) return MOE_ERR_INVALID_ARG;
  return ep_signal_impl(flags_host, rank, P, epoch, ws, wait_limit_ns, (cudaStream_t)stream);
}

moe_status moe_ep_home_combine(const moe_shape* s, const void* y_back, const int32_t* slot_send_row,
                               int64_t send_rows, void* y, moe_stream_t stream) {
  moe_status r = check_shape(s);
  if (r != MOE_OK) return r;
  if (s->ep < 2 || send_rows < 0) return MOE_ERR_INVALID_ARG;
  if (s->T == 0) return MOE_OK;
  if (!y_back || !slot_send_row || !y || send_rows == 0) return MOE_ERR_INVALID_ARG;
  if (!aligned(y_back, 16) || !aligned(y, 16) || !aligned(slot_send_row, 4))
    return MOE_ERR_ALIGNMENT;
  return cuda_status(launch_ep_home_combine(s->dtype, y_back, slot_send_row, y, s->T, s->d, s->k,
                                            send_rows, (cudaStream_t)stream));
}

moe_status moe_dispatch_layout(const moe_shape* s, const int32_t* topk_idx,
                               const int32_t* expert_rank_host, const moe_layout* out, void* ws,
                               size_t ws_bytes, moe_stream_t stream) {
  return layout_entry(s, topk_idx, expert_rank_host, out, ws, ws_bytes, -1, kWaitLimitNs,
                      (cudaStream_t)stream);
}

moe_status moe_debug_dispatch_layout_stall(const moe_shape* s, const int32_t* topk_idx,
                                           const int32_t* expert_rank_host, const moe_layout* out,
                                           void* ws, size_t ws_bytes, int32_t stall_block,
                                           int64_t wait_limit_ns, moe_stream_t stream) {
  if (wait_limit_ns <= 0 || wait_limit_ns > kWaitLimitNs) return MOE_ERR_INVALID_ARG;
  return layout_entry(s, topk_idx, expert_rank_host, out, ws, ws_bytes, stall_block,
                      wait_limit_ns, (cudaStream_t)stream);
}

moe_status moe_permute(const moe_shape* s, const void* x, const int32_t* row_token, void* x_perm,
                       moe_stream_t stream) {
  moe_status r = check_shape(s);
  if (r != MOE_OK) return r;
  if (s->T == 0) return MOE_OK;
  if (!x || !row_token || !x_perm) return MOE_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(x_perm, 16) || !aligned(row_token, 4)) return MOE_ERR_ALIGNMENT;
  return cuda_status(launch_permute(x, row_token, nullptr, x_perm, s->T, s->k,
                                    (uint32_t)(s->d * esize(s->dtype)), (cudaStream_t)stream));
}

moe_status moe_permute_by_token(const moe_shape* s, const void* x, const int32_t* slot_row,
                                void* x_perm, moe_stream_t stream) {
  moe_status r = check_shape(s);
  if (r != MOE_OK) return r;
  if (s->T == 0) return MOE_OK;
  if (!x || !slot_row || !x_perm) return MOE_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(x_perm, 16) || !aligned(slot_row, 4)) return MOE_ERR_ALIGNMENT;
  return cuda_status(launch_permute(x, nullptr, slot_row, x_perm, s->T, s->k,
                                    (uint32_t)(s->d * esize(s->dtype)), (cudaStream_t)stream));
}

moe_status moe_grouped_swiglu(const moe_shape* s, const void* x_perm, const int32_t* offsets,
                              const void* packed, void* h, void* y_perm, void* ws, size_t ws_bytes,
                              moe_stream_t stream) {
  return moe_debug_grouped_swiglu_engine(s, x_perm, nullptr, offsets, packed, h, y_perm, ws,
                                         ws_bytes, kEngineAuto, stream);
}

moe_status moe_debug_grouped_swiglu_engine(const moe_shape* s, const void* a_rows,
                                           const int32_t* row_token, const int32_t* offsets,
                                           const void* packed, void* h, void* y_perm, void* ws,
                                           size_t ws_bytes, int32_t engine, moe_stream_t stream) {
  if (engine < kEngineAuto || engine > kEnginePairGateUp) return MOE_ERR_INVALID_ARG;
  if (row_token)
    return gather_impl(s, a_rows, row_token, offsets, packed, h, y_perm, ws, ws_bytes, engine,
                       (cudaStream_t)stream);
  const void* x_perm = a_rows;
  moe_status r = check_shape(s);
  if (r != MOE_OK) return r;
  if (s->T == 0) return MOE_OK;
  if (!x_perm || !offsets || !packed || !h || !y_perm || !ws) return MOE_ERR_INVALID_ARG;
  if (!aligned(x_perm, 16) || !aligned(h, 16) || !aligned(y_perm, 16) || !aligned(offsets, 4) ||
      !aligned(packed, kAlign) || !aligned(ws, kAlign))
    return MOE_ERR_ALIGNMENT;
  if (ws_bytes < scratch_bytes(s)) return MOE_ERR_WORKSPACE;
  Packed pk = carve_packed(s, packed);
  return do_grouped(s, x_perm, offsets, &pk, h, y_perm, carve_scratch(s, ws).ctl,
                    (cudaStream_t)stream, engine);
}

moe_status moe_combine(const moe_shape* s, const void* y_perm, const int32_t* slot_row,
                       const float* gate, void* y, moe_stream_t stream) {
  moe_status r = check_shape(s);
  if (r != MOE_OK) return r;
  if (s->T == 0) return MOE_OK;
  if (!y_perm || !slot_row || !y) return MOE_ERR_INVALID_ARG;
  if (!aligned(y_perm, 16) || !aligned(y, 16) || !aligned(slot_row, 4) || (gate && !aligned(gate, 4)))
    return MOE_ERR_ALIGNMENT;
  return cuda_status(
      launch_combine(s->dtype, y_perm, slot_row, gate, y, s->T, s->d, s->k, (cudaStream_t)stream));
}

moe_status moe_forward(const moe_shape* s, const void* x, const void* packed, const float* bias,
                       const int32_t* expert_rank_host, void* y, const moe_forward_buffers* buffers,
                       void* ws, size_t ws_bytes, moe_stream_t stream) {
  return forward_impl(s, x, packed, bias, expert_rank_host, y, buffers, ws, ws_bytes,
                      (cudaStream_t)stream, nullptr);
}

moe_status moe_debug_forward_options(const moe_shape* s, const void* x, const void* packed,
                                     const float* bias, const int32_t* expert_rank_host, void* y,
                                     const moe_forward_buffers* buffers, void* ws, size_t ws_bytes,
                                     int32_t options, moe_stream_t stream) {
  if (options & ~MOE_FWD_COMBINE_IN_DOWN) return MOE_ERR_INVALID_ARG;
  return forward_impl(s, x, packed, bias, expert_rank_host, y, buffers, ws, ws_bytes,
                      (cudaStream_t)stream, nullptr, false, nullptr, nullptr, nullptr, options);
}

moe_status moe_forward_selection_bias(const moe_shape* s, const void* x, const void* packed,
                                      const float* bias, const float* selection_bias,
                                      const int32_t* expert_rank_host, void* y,
                                      const moe_forward_buffers* buffers, void* ws,
                                      size_t ws_bytes, moe_stream_t stream) {
  if (!selection_bias) return MOE_ERR_INVALID_ARG;
  return forward_impl(s, x, packed, bias, expert_rank_host, y, buffers, ws, ws_bytes,
                      (cudaStream_t)stream, nullptr, false, nullptr, nullptr, selection_bias);
}

moe_status moe_forward_routed(const moe_shape* s, const void* x, const void* packed,
                              const int32_t* topk_idx, const float* topk_gate,
                              const int32_t* expert_rank_host, void* y,
                              const moe_forward_buffers* buffers, void* ws, size_t ws_bytes,
                              moe_stream_t stream) {
  return forward_impl(s, x, packed, nullptr, expert_rank_host, y, buffers, ws, ws_bytes,
                      (cudaStream_t)stream, nullptr, true, topk_idx, topk_gate);
}

moe_status moe_forward_timed(const moe_shape* s, const void* x, const void* packed,
                             const float* bias, const int32_t* expert_rank_host, void* y,
                             const moe_forward_buffers* buffers, void* ws, size_t ws_bytes,
                             moe_event_t* events, moe_stream_t stream) {
  if (!events) return MOE_ERR_INVALID_ARG;
  for (int i = 0; i <= MOE_FORWARD_STAGES; ++i)
    if (!events[i]) return MOE_ERR_INVALID_ARG;
  return forward_impl(s, x, packed, bias, expert_rank_host, y, buffers, ws, ws_bytes,
                      (cudaStream_t)stream, reinterpret_cast<cudaEvent_t*>(events));
}

moe_status moe_grouped_swiglu_gather(const moe_shape* s, const void* x, const int32_t* row_token,
                                     const int32_t* offsets, const void* packed, void* h,
                                     void* y_perm, void* ws, size_t ws_bytes, moe_stream_t stream) {
  return gather_impl(s, x, row_token, offsets, packed, h, y_perm, ws, ws_bytes, kEngineAuto,
                     (cudaStream_t)stream);
}

moe_status moe_get_device_status(void* ws, moe_stream_t stream, moe_status* out) {
  if (!ws || !out) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  if (cudaStreamSynchronize(st) != cudaSuccess) return MOE_ERR_CUDA;
  uint32_t v = 0;
  if (cudaMemcpy(&v, ws, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
  *out = (moe_status)v;
  if (v != MOE_OK) {
    if (cudaMemsetAsync(ws, 0, sizeof(uint32_t), st) != cudaSuccess) return MOE_ERR_CUDA;
    // the detail word (offset 4) is informational; clear it with the status
    if (cudaMemsetAsync(static_cast<uint8_t*>(ws) + 4, 0, sizeof(uint32_t), st) != cudaSuccess)
      return MOE_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

}  // extern "C"
