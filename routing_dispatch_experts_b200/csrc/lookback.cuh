// lookback.cuh - decoupled-lookback exclusive scan across blocks, shared by
// the layout histogram kernel and the fused router kernel.
//
// Block b (its index taken from a ticket counter, so it only ever waits on
// blocks that started before it) publishes each bin's count as an
// "aggregate", walks back over its predecessors adding their aggregates
// until one has published an "inclusive prefix", then publishes its own
// inclusive prefix.  One 64-bit word per (block, bin) holds flag and value,
// so a reader sees both together.  Waits give up after `limit_ns`; a block
// that gives up records MOE_ERR_DEVICE_TIMEOUT and publishes an error flag so
// its successors stop at once.  The words must be zero when the scan starts;
// the layout scatter kernel, the one reader of the results, zeroes each
// block's words after reading them, so a workspace stays ready for the next
// call of any shape.
#pragma once

#include "kernels.cuh"

namespace moe {

constexpr uint32_t kFlagNone = 0, kFlagAgg = 1, kFlagIncl = 2, kFlagErr = 3;

__device__ __forceinline__ void lb_publish(uint64_t* w, uint32_t flag, uint32_t value) {
  atomicExch(reinterpret_cast<unsigned long long*>(w),
             ((unsigned long long)flag << 32) | (unsigned long long)value);
}

__device__ __forceinline__ uint64_t lb_poll(const uint64_t* w) {
  return *reinterpret_cast<const volatile unsigned long long*>(w);
}

// One bin of the scan for block b: returns false on time-out / error.
// `publish_self` = false models a block that never publishes (test hook).
// Predecessors are read kLookbackWindow at a time with independent loads,
// so a block far from the last inclusive prefix needs few round trips.
constexpr int kLookbackWindow = 8;

__device__ __forceinline__ bool lookback_bin(uint64_t* status, int bins, int b, int bin,
                                             uint32_t agg, bool publish_self, int64_t limit_ns,
                                             uint32_t* excl_out) {
  uint64_t* mine = status + (size_t)b * bins + bin;
  uint32_t excl = 0;
  if (b > 0) {
    if (publish_self) lb_publish(mine, kFlagAgg, agg);
    int q = b - 1;
    bool done = false;
    while (!done && q >= 0) {
      const int n = q + 1 < kLookbackWindow ? q + 1 : kLookbackWindow;
      uint64_t w[kLookbackWindow];
#pragma unroll
      for (int i = 0; i < kLookbackWindow; ++i)
        if (i < n) w[i] = lb_poll(status + (size_t)(q - i) * bins + bin);
#pragma unroll
      for (int i = 0; i < kLookbackWindow; ++i) {
        if (i >= n || done) continue;
        uint64_t v = w[i];
        if ((uint32_t)(v >> 32) == kFlagNone) {
          const uint64_t* src = status + (size_t)(q - i) * bins + bin;
          const uint64_t ts = globaltimer_ns();
          do {
            __nanosleep(32);
            v = lb_poll(src);
            if ((uint32_t)(v >> 32) != kFlagNone) break;
          } while (globaltimer_ns() - ts <= (uint64_t)limit_ns);
          if ((uint32_t)(v >> 32) == kFlagNone) {
            if (publish_self) lb_publish(mine, kFlagErr, 0);
            return false;
          }
        }
        const uint32_t fl = (uint32_t)(v >> 32);
        if (fl == kFlagErr) {
          if (publish_self) lb_publish(mine, kFlagErr, 0);
          return false;
        }
        excl += (uint32_t)v;
        if (fl == kFlagIncl) done = true;
      }
      q -= n;
    }
  }
  if (publish_self) lb_publish(mine, kFlagIncl, excl + agg);
  *excl_out = excl;
  return true;
}

// Count one token into a shared histogram: its k experts, its distinct
// ranks, and the two statistic bins at the end (tokens whose experts sit on
// one rank; assignments on the token's home rank floor(t * ep / T)).
// Registers only: the distinct-rank test compares against the token's
// earlier slots.  s_map is the expert -> rank map in shared memory.
template <int KMAX>
__device__ __forceinline__ void count_token(const int (&e)[KMAX], int k, int64_t t, int64_t T, int E,
                                            int ep, const uint8_t* s_map, int* hist, int* single,
                                            int* home) {
  const int home_r = (int)((t * ep) / T);
  int r[KMAX];
  int nr = 0;
#pragma unroll
  for (int j = 0; j < KMAX; ++j) {
    if (j < k) {
      atomicAdd(&hist[e[j]], 1);
      r[j] = ep > 1 ? (int)s_map[e[j]] : 0;
      *home += r[j] == home_r;
      bool seen = false;
#pragma unroll
      for (int q = 0; q < j; ++q) seen |= r[q] == r[j];
      if (!seen) {
        ++nr;
        if (ep > 1) atomicAdd(&hist[E + r[j]], 1);
      }
    }
  }
  *single += nr == 1;
}

}  // namespace moe
