// Split-KV schedule shared by the decode split kernels and the combine kernel.
//
// The pages of all sequences are laid end to end on a cost axis (sequence 0's
// pages, then sequence 1's, ...), each non-empty sequence preceded by
// `piece_cost` units that hold no page: the time a worker spends starting and
// finishing a piece (query load, partial write, pipeline refill), in pages.
// That axis is cut into contiguous chunks of `chunk` units; worker w takes the
// pages at positions [w*chunk, (w+1)*chunk).  A worker's chunk may end inside
// one sequence and continue into the next, and a worker whose chunk crosses a
// sequence start is given correspondingly fewer pages.  Each overlap of a
// worker with a sequence's pages is a "piece"; a piece writes one partial
// result (softmax-normalised latent output and log-sum-exp per row) to the
// workspace.  The pieces of sequence b are consecutive: piece_begin[b] ..
// piece_begin[b] + npieces[b] - 1, worker w's piece of b being piece_begin[b] +
// (w - w_first[b]).  With chunk >= ceil(total / G) at most G workers are busy,
// so there are at most G + batch - 1 pieces.
//
// Every CTA rebuilds this schedule from seq_lens in shared memory (two block
// scans over the batch), so no planning launch and no metadata buffer exist.
//
// Context split: with kv_ranks > 1 (one call per rank, e.g. one per GPU) rank r
// takes only the window [P_b r / R, P_b (r + 1) / R) of sequence b's P_b pages;
// the schedule above is built over the windows, and page indices stay absolute
// (the window's first page is added back), so masking and the page table are unchanged.
#pragma once

#include "common.cuh"

namespace mla {

constexpr int kMaxBatch = 1024;   // sequences per decode call
constexpr int kMinChunk = 4;      // pages: keeps per-piece overhead bounded

struct PlanSmem {
  int start[kMaxBatch + 1];        // cost-axis position of each sequence's first page; start[B] = total
  int npg[kMaxBatch];              // pages of each sequence (in this rank's window)
  uint16_t piece_begin[kMaxBatch + 1];  // first piece of each sequence; piece_begin[B] = #pieces
                                       // (at most workers + batch, well below 2^16)
  int chunk;                       // cost units per worker
  // what the window of a sequence is computed from (see plan_win0)
  const int32_t* seq_lens;
  int nq, max_pages, page_size, kv_rank, kv_ranks;
  int warp_tot[32];
};

// Host-side bound on the number of pieces, used for workspace sizing.
inline int64_t max_pieces(int G, int batch) { return (int64_t)G + batch; }

// Number of pages of sequence b; 0 (and a recorded range error) when its
// length is outside [nq, max_pages * page_size].
__device__ __forceinline__ int seq_pages(const int32_t* seq_lens, int b, int nq, int max_pages,
                                         int page_size, int32_t* dev_status) {
  int len = seq_lens[b];
  if (len < nq || len > max_pages * page_size) {
    record_status(dev_status, MLA_ERR_RANGE);
    return 0;
  }
  return (len + page_size - 1) / page_size;
}

// Block-wide exclusive scan of one int per thread; returns the exclusive prefix
// and writes the block total to *total.  All threads of the block must call it.
__device__ __forceinline__ int block_exclusive_scan(int v, int* warp_tot, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nwarps = (blockDim.x + 31) >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_tot[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int t = lane < nwarps ? warp_tot[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    warp_tot[lane] = t;  // inclusive prefix of warp totals
  }
  __syncthreads();
  int excl = x - v + (warp > 0 ? warp_tot[warp - 1] : 0);
  *total = warp_tot[nwarps - 1];
  __syncthreads();
  return excl;
}

// First page of rank r's window over n pages (R ranks): floor(n r / R).
__device__ __forceinline__ int window_begin(int n, int r, int R) { return (int)(((long long)n * r) / R); }

// First page of sequence b's window (0 without a context split).
__device__ __forceinline__ int plan_win0(const PlanSmem* ps, int b) {
  if (ps->kv_ranks == 1) return 0;
  const int len = ps->seq_lens[b];
  const int pages = (len < ps->nq || len > ps->max_pages * ps->page_size) ? 0 : (len + ps->page_size - 1) / ps->page_size;
  return window_begin(pages, ps->kv_rank, ps->kv_ranks);
}

// Fills ps->start, ps->npg, ps->piece_begin, ps->chunk and the window parameters for
// `batch` sequences and G workers, over the windows of rank kv_rank of kv_ranks.
__device__ __forceinline__ void build_plan(PlanSmem* ps, const int32_t* seq_lens, int batch, int nq, int max_pages,
                           int page_size, int G, int piece_cost, int32_t* dev_status, int kv_rank = 0,
                           int kv_ranks = 1) {
  // pass 1: pages per sequence (in this rank's window) -> cost-axis positions
  int carry = 0;
  for (int base = 0; base < batch; base += blockDim.x) {
    int b = base + threadIdx.x;
    int v = b < batch ? seq_pages(seq_lens, b, nq, max_pages, page_size,
                                  blockIdx.x == 0 && blockIdx.y == 0 ? dev_status : nullptr)
                      : 0;
    if (b < batch) v = window_begin(v, kv_rank + 1, kv_ranks) - window_begin(v, kv_rank, kv_ranks);
    const int lead = v > 0 ? piece_cost : 0;
    int tot;
    int ex = block_exclusive_scan(v + lead, ps->warp_tot, &tot);
    if (b < batch) {
      ps->start[b] = carry + ex + lead;
      ps->npg[b] = v;
    }
    carry += tot;
  }
  if (threadIdx.x == 0) {
    ps->start[batch] = carry;
    int c = (carry + G - 1) / G;
    ps->chunk = c < kMinChunk ? kMinChunk : c;
    ps->seq_lens = seq_lens;
    ps->nq = nq;
    ps->max_pages = max_pages;
    ps->page_size = page_size;
    ps->kv_rank = kv_rank;
    ps->kv_ranks = kv_ranks;
  }
  __syncthreads();
  const int chunk = ps->chunk;
  // pass 2: pieces per sequence -> piece_begin
  carry = 0;
  for (int base = 0; base < batch; base += blockDim.x) {
    int b = base + threadIdx.x;
    int v = 0;
    if (b < batch) {
      const int s = ps->start[b], n = ps->npg[b];
      v = n > 0 ? (s + n - 1) / chunk - s / chunk + 1 : 0;
    }
    int tot;
    int ex = block_exclusive_scan(v, ps->warp_tot, &tot);
    if (b < batch) ps->piece_begin[b] = (uint16_t)(carry + ex);
    carry += tot;
  }
  if (threadIdx.x == 0) ps->piece_begin[batch] = (uint16_t)carry;
  __syncthreads();
}

// The last sequence whose first page lies at or before cost position f (0 if
// none); f < total.  Its pages may end before f: the iterator skips ahead.
__device__ __forceinline__ int seq_at_position(const PlanSmem* ps, int batch, int f) {
  int lo = 0, hi = batch - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (ps->start[mid] <= f) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// One (sequence, page range) overlap of this worker's chunk.
struct Piece {
  int b, pg_begin, pg_end, id;
};

// Iterates the pieces of worker w in order; identical in every role.
struct PieceIter {
  const PlanSmem* ps;
  int batch, w, chunk, f, f1, b;
  __device__ PieceIter(const PlanSmem* ps_, int batch_, int w_) : ps(ps_), batch(batch_), w(w_) {
    chunk = ps->chunk;
    const int total = ps->start[batch];
    f = w * chunk;
    f1 = min(f + chunk, total);
    b = f < f1 ? seq_at_position(ps, batch, f) : 0;
  }
  __device__ bool next(Piece* p) {
    // skip empty sequences and those whose pages end before f
    while (b < batch && (ps->npg[b] == 0 || ps->start[b] + ps->npg[b] <= f)) ++b;
    if (b >= batch) return false;
    const int sb = ps->start[b];
    const int s = max(f, sb);
    if (s >= f1) return false;
    const int e = min(f1, sb + ps->npg[b]);
    const int w0 = plan_win0(ps, b);
    p->b = b;
    p->pg_begin = s - sb + w0;   // absolute page indices of the sequence
    p->pg_end = e - sb + w0;
    p->id = ps->piece_begin[b] + (w - sb / chunk);
    f = e;
    return true;
  }
};

}  // namespace mla
