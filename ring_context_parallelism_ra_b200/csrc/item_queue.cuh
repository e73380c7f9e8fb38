// Hand-out of work items to the roles of a persistent CTA (shared by the
// forward and backward tensor-core kernels).
#pragma once

#include <stdint.h>

#include "common.cuh"
#include "ptx.cuh"

namespace ra {

// Work items of the persistent attention kernels are handed out one at a
// time from a global counter, in each kernel's order of items.  A static
// deal (item round * CTAs + c to CTA c) lets a CTA on a slower SM fall
// further behind with every round, until the CTAs running together are on
// different KV heads and no longer share their K/V tiles or dQ lines in L2;
// taken from a counter, the items in flight are always the next ~CTAs of the
// order.  The producer takes each item and publishes its index to the CTA's
// other roles through a small ring in shared memory.
constexpr int kItemSlots = 4;
struct ItemQueue {
  volatile int* slot;  // [kItemSlots] item index, -1 = no more items
  uint64_t* full;      // [kItemSlots] 1 arrival: the producer published
  uint64_t* empty;     // [kItemSlots] one arrival per consumer thread
};

// Producer: take the next item for `round`.  Returns its index, -1 when the
// items are exhausted (published as well), -2 if a wait gave up.
__device__ __forceinline__ int item_publish(const ItemQueue& q, unsigned int* counter, int items,
                                            int round, const DevCtx& ctx, volatile int* abort) {
  const int sl = round % kItemSlots;
  if (!mbar_wait(&q.empty[sl], ((round / kItemSlots) & 1) ^ 1, ctx, abort)) return -2;
  const unsigned int t = atomicAdd(counter, 1u);
  const int idx = t < static_cast<unsigned int>(items) ? static_cast<int>(t) : -1;
  q.slot[sl] = idx;
  mbar_arrive(&q.full[sl]);  // release: the index is visible to the waiters
  return idx;
}

// Consumer: the item of `round` as the producer published it (-1: none left,
// -2: a wait gave up).
__device__ __forceinline__ int item_take(const ItemQueue& q, int round, const DevCtx& ctx,
                                         volatile int* abort) {
  const int sl = round % kItemSlots;
  if (!mbar_wait(&q.full[sl], (round / kItemSlots) & 1, ctx, abort)) return -2;
  const int idx = q.slot[sl];
  mbar_arrive(&q.empty[sl]);
  return idx;
}

}  // namespace ra
