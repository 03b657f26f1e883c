// Pieces the two tcgen05 split-KV attention kernels share: the page-id
// cursor of the TMA producer and the lazy-rescale threshold of the online
// softmax.
#pragma once

#include "common.cuh"

namespace mlra {

constexpr float kRescaleLog2 = 8.f;       // O is rescaled only when the running max grows by more than 2^8
constexpr int kIdAhead = 8;               // page ids read this many pages before their tile
constexpr int kIdRing = 16;
static_assert(kIdRing >= kIdAhead + 2, "id ring holds the ids in flight");

// Cursor over a worker's pages in walk order that reads each page's id from
// the page table (the producer runs one of these ahead of its loads).
struct IdFetch {
  SegWalk w;
  int p;
  bool live;
  __device__ __forceinline__ IdFetch(const WorkerPlan& plan, int B, int maxL, const int* seq_lens)
      : w(plan, B, maxL), p(0), live(false) {
    live = w.next(seq_lens);
    if (live) p = w.pg0;
  }
  __device__ __forceinline__ void step(const int* seq_lens) {
    if (++p >= w.pg1) {
      live = w.next(seq_lens);
      if (live) p = w.pg0;
    }
  }
  // id of the current page (not yet waited for), then advance
  __device__ __forceinline__ int fetch(const int* seq_lens, const int* page_table, int maxp) {
    const int id = __ldg(page_table + (size_t)w.b * maxp + p);
    step(seq_lens);
    return id;
  }
};

}  // namespace mlra
