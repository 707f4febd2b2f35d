// checks.cuh - host-side argument checks shared by every entry point of the
// C ABI, so that entry points taking the same arguments accept and reject
// exactly the same inputs.
#pragma once

#include <algorithm>
#include <cstdint>
#include <cstring>

#include "kernels.cuh"

namespace moe {

inline int esize(int dtype) { return dtype == MOE_BF16 ? 2 : 4; }

inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// The problem statement's limits (include/moe.h, moe_shape): invalid shapes
// give MOE_ERR_INVALID_ARG, valid shapes outside the kernels' coverage
// MOE_ERR_UNSUPPORTED.
inline moe_status check_shape(const moe_shape* s) {
  if (!s) return MOE_ERR_INVALID_ARG;
  if (s->dtype != MOE_F32 && s->dtype != MOE_BF16) return MOE_ERR_INVALID_ARG;
  if (s->T < 0 || s->E < 1 || s->E > 256 || s->k < 1 || s->k > std::min(s->E, 16) || s->ep < 1 ||
      s->ep > s->E || s->E % s->ep != 0 || s->d <= 0 || s->f <= 0)
    return MOE_ERR_INVALID_ARG;
  if (s->T * (int64_t)s->k >= (int64_t(1) << 31)) return MOE_ERR_INVALID_ARG;
  if (s->d % 64 != 0 || s->f % 64 != 0 || (int64_t)s->d * esize(s->dtype) > 16384)
    return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

// The output arrays of a dispatch layout: present where the shape needs
// them (with T == 0 the per-assignment arrays are empty and may be NULL;
// the send layout only when ep > 1), 4-byte aligned, stats 8-byte aligned.
inline moe_status check_layout_ptrs(const moe_shape* s, const moe_layout* o) {
  const bool rows = s->T > 0;
  if (!o || !o->expert_counts || !o->expert_offsets || (rows && (!o->row_token || !o->slot_row)))
    return MOE_ERR_INVALID_ARG;
  if (s->ep > 1 && (!o->rank_counts || !o->rank_offsets ||
                    (rows && (!o->send_token || !o->slot_send_row))))
    return MOE_ERR_INVALID_ARG;
  const void* ps[] = {o->expert_counts, o->expert_offsets, o->row_token, o->slot_row,
                      o->rank_counts, o->rank_offsets, o->send_token, o->slot_send_row};
  for (const void* p : ps)
    if (p && !aligned(p, 4)) return MOE_ERR_ALIGNMENT;
  if (o->stats && !aligned(o->stats, 8)) return MOE_ERR_ALIGNMENT;
  return MOE_OK;
}

// Expert -> rank map from the caller's host array (NULL = contiguous
// placement e -> e / (E/ep)).  A placement must be a partition in which every
// rank owns exactly E/ep experts ("Expert Coupling in MoE Pretraining",
// Table III: P ranks holding the E experts); anything else is
// MOE_ERR_INVALID_ARG.
inline moe_status build_map(const moe_shape* s, const int32_t* host_map, RankMap* m) {
  std::memset(m, 0, sizeof(*m));
  const int per = s->E / s->ep;
  if (!host_map) {
    for (int e = 0; e < s->E; ++e) m->r[e] = (uint8_t)(e / per);
    return MOE_OK;
  }
  int count[256] = {0};
  for (int e = 0; e < s->E; ++e) {
    const int r = host_map[e];
    if (r < 0 || r >= s->ep) return MOE_ERR_INVALID_ARG;
    ++count[r];
    m->r[e] = (uint8_t)r;
  }
  for (int r = 0; r < s->ep; ++r)
    if (count[r] != per) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

}  // namespace moe
