// Split-KV latent attention on CTA pairs with 2-SM tensor-core instructions
// (tcgen05 .cta_group::2, TMEM, TMA): exact fp32 scores, nothing but the MMA
// operands crosses the pair.
//
// Shape: d_c = 512, d_rope = 64 (576-wide cache rows), 64-token pages, a tile of up
// to 128 query rows (query token, head) per CTA pair.  CTA c of the pair owns rows
// [64c, 64c + 64) of the tile: its part of the query, its rows of the scores, its
// softmax and its rows of the latent output.  One MMA issued by CTA 0 computes
// both CTAs' rows; its B operand is split by columns, each CTA supplying half from
// its own shared memory at the same offset.
//
// A step is 2 pages (128 keys); CTA c's page is page c of the step.
//   scores  S[128 x 128] = Q[128 x 576] . K[128 x 576]^T   (M = 128 rows, N = 128 keys)
//           B = the two pages at full width, CTA c supplying its own page (loaded
//           by TMA into a step buffer: 9 blocks [64 keys x 64 columns]).  Every page
//           crosses HBM once and each CTA receives complete 576-wide dot products.
//   softmax per row, in the CTA that owns it (four threads per row: two pages times
//           two halves of the page's keys).  P is double-buffered: block 0 (the keys
//           of page 0) in the step buffer's rope block, which the scores no longer
//           need, block 1 in a P block of its own per step parity; so the softmax of
//           step t + 1 does not wait for the value MMAs of step t.
//   values  O[128 x 512] += P[128 x 128] . C[128 x 512]  (N = 256 latent columns per
//           MMA).  B is split by columns: for the keys of page p, CTA c supplies
//           latent columns [256j + 128c, +128) at blocks 4j + 2p, 4j + 2p + 1 of the
//           step buffer.  For its own page those blocks already hold exactly these
//           columns (block b holds columns 64b).  For the peer's page they held the
//           other half of its own page, which the scores no longer need: once the
//           step's score MMAs are done, a loader warp overwrites them with the peer
//           page's columns [256j + 128c, +128), read from L2 by TMA (the peer just
//           loaded that page); where a page is partial, per-thread copies fill slots
//           past the sequence's end with zeros instead.  So each CTA reads 72 KB per
//           step from HBM and 32 KB from L2.  The value MMAs run page by page; once
//           page 0's are done, the blocks they read (0, 1, 4, 5 and 8) are reloaded
//           for the step two ahead, the other four when page 1's are done.
//
// TMEM (512 columns, same map in both CTAs; a pair tile with M = 128 folds each
// CTA's 64 rows into the 128 lanes: lanes [0,64) hold the first N/2 columns, lanes
// [64,128) the rest):
//   [0,64), [64,128)  S of steps t even / odd (page 0 of the step in lanes 0-63,
//                     page 1 in lanes 64-127)
//   [128,256)         latent columns [0,256) of this CTA's query rows (bf16 pairs),
//                     A of the first 16 score MMAs (lanes r and r + 64 hold row r);
//                     columns [256,576) of the query stay in shared memory
//   [256,512)         O: latent 256j + [0,128) in lanes 0-63, 256j + [128,256) in
//                     lanes 64-127, j = 0 at [256,384), j = 1 at [384,512)
//
// Warps (416 threads per CTA): 0 loads the query and the step buffers (TMA), 1 owns
// TMEM and, in CTA 0, issues the score MMAs, 12 (CTA 0) issues the value MMAs, 2
// fetches the peer half, 3 hands a half fetched by per-thread copies to the value
// issuer, 4-11 run the softmax and the epilogue (warps w and w + 4 share TMEM lane
// quarter w & 3, each reading half of the columns).  Each MMA warp runs converged
// and one elected lane issues (an MMA issued from a lone lane under data-dependent
// control flow costs several times its execution time).  The running max is only moved (and O rescaled in TMEM) when it grows by more than
// 2^8.  No global load is outstanding at a release arrive on the softmax's path (a
// release waits for it): page ids and lengths are read a step ahead.  Every
// mbarrier wait is bounded: on time-out the kernel records MLA_ERR_TIMEOUT, stops
// its loops, drains its MMAs and frees TMEM.
#include <cuda.h>

#include "common.cuh"
#include "decode.h"
#include "plan.cuh"
#include "sm100.cuh"

namespace mla {

namespace {

using namespace sm100;

constexpr int kThreads = 416;
constexpr int kStepPages = 2;
constexpr int kBlockBytes = 8192;             // [64 keys x 64 columns] bf16, 128-byte swizzle
constexpr int kBufBytes = 9 * kBlockBytes;    // a step buffer: the own page at full width
constexpr int kQBytes = 5 * kBlockBytes;      // query columns [256,576) of 64 rows
constexpr int kPBytes = 2 * kBlockBytes;      // block 1 of P [64 rows x 128 keys] of steps t even / odd
constexpr int kOffQ = 0;
constexpr int kOffP = kOffQ + kQBytes;
constexpr int kOffBuf = kOffP + kPBytes;
constexpr int kOffXch = kOffBuf + 2 * kBufBytes;           // row maxima [2][2][128], row sums [2][128] (fp32)
constexpr int kOffPlan = kOffXch + 6 * 128 * 4;
constexpr int kOffBar = kOffPlan + ((int(sizeof(PlanSmem)) + 15) & ~15);
constexpr int kNumBars = 32;
constexpr int kOffMisc = kOffBar + kNumBars * 8;           // TMEM base, abort flag
constexpr int kSmemBytes = kOffMisc + 64 + 1024;           // + 1 KB alignment slack
constexpr float kRescaleThreshold = 8.0f;     // log2 units
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemQ = 128;
constexpr uint32_t kTmemO = 256;
constexpr long long kDrainCycles = 1ll << 24;

static_assert(kSmemBytes <= 232448, "shared memory budget");
static_assert(kOffP % 1024 == 0 && kOffBuf % 1024 == 0 && kBufBytes % 1024 == 0, "swizzle alignment");

struct PairParams {
  DecodeArgs d;
  int rows_total;   // nq * H
  float scale_log2; // softmax scale * log2(e)
  long long spin_limit;
};

struct Bars {
  uint64_t kfull[2];    // CTA 0: both CTAs' pages of a step landed in the step buffer (2 arrivals + bytes)
  uint64_t buf_lo[2];   // both: the step's value MMAs of page 0 are done (blocks 0, 1, 4, 5, 8 of its buffer)
  uint64_t buf_free[2]; // both: the step's value MMAs are done with its buffer
  uint64_t vland[2];    // local: per-thread peer-half copies of a partial step have landed (32 arrivals)
  uint64_t vfull[2];    // CTA 0: both CTAs' step buffers hold the value operand (2 arrivals)
  uint64_t q_full;      // CTA 0: the shared-memory part of both query halves loaded (2 arrivals + bytes)
  uint64_t qt_full;     // CTA 0: the TMEM part of the query written by the 16 softmax warps of the pair
  uint64_t q_empty;     // both: the piece's score MMAs are done with the query tile
  uint64_t s_full[2];   // both: scores of a step are in TMEM (and its buffer's other half is free)
  uint64_t s_empty[2];  // CTA 0: the 16 softmax warps of the pair have read them
  uint64_t p_full[2];   // CTA 0: P of a step written (and O rescaled) in both CTAs
  uint64_t p_empty[2];  // both: the value MMAs of a step are done (O current); [t & 1] for step t, so
                        // that a waiter (P no longer waits for them) is never two phases behind
  uint64_t o_free;      // CTA 0: the epilogue of a piece has read O in both CTAs
  uint64_t drain;       // both: every MMA issued has completed (a commit from each of the two issuers)
  uint64_t xm, xl;      // local: the 8 softmax warps published a step's row maxima / a piece's row sums
};
static_assert(sizeof(Bars) <= kNumBars * 8, "barrier area");

// A step: up to 2 consecutive pages of one piece.  Every role walks the same steps.
struct Step {
  int b;         // sequence
  int pg0;       // first page of the step (page index within the sequence)
  int np;        // pages in the step (1 or 2)
  int id;        // workspace slot of the piece
  int p;         // index of the piece among this worker's pieces
  bool first, last;
};

struct StepCursor {
  PieceIter it;
  Piece pc;
  int pg = 0, p = -1;
  bool in_piece = false;
  __device__ StepCursor(const PlanSmem* ps, int batch, int w) : it(ps, batch, w) {}
  __device__ bool next(Step* s) {
    if (!in_piece || pg >= pc.pg_end) {
      if (!it.next(&pc)) return false;
      in_piece = true;
      pg = pc.pg_begin;
      ++p;
    }
    s->b = pc.b;
    s->pg0 = pg;
    s->np = min(kStepPages, pc.pg_end - pg);
    s->id = pc.id;
    s->p = p;
    s->first = pg == pc.pg_begin;
    pg += s->np;
    s->last = pg >= pc.pg_end;
    return true;
  }
};

// Physical page of page `pg` of sequence b, or -1 (and a recorded range error)
// when the page table names a page outside the pool.
__device__ __forceinline__ int page_id(const DecodeArgs& a, int b, int pg, int32_t* status) {
  const int id = a.page_table[(size_t)b * a.max_pages + pg];
  if (id < 0 || id >= a.num_pages) {
    record_status(status, MLA_ERR_RANGE);
    return -1;
  }
  return id;
}

// What the value operand of a step needs from memory in CTA c: the peer's page
// (id_p, or -1 when the step has no such page or it lies outside the pool) with
// nv_p valid keys, and the number of valid keys of the own page (64 when the own
// page is missing: its slots were zero-filled by the load).  `full` when both pages
// are complete, so that the peer half can be copied whole by TMA; otherwise slots
// past the sequence's end are zeroed with per-thread copies.
struct PeerFetch {
  int id_p, nv_p, nv_o;
  bool full;
};
__device__ __forceinline__ PeerFetch peer_fetch(const DecodeArgs& a, int b, int pg0, int np, int c) {
  PeerFetch f;
  const int len = a.seq_lens[b];
  const int pp = 1 - c;
  f.id_p = pp < np ? page_id(a, b, pg0 + pp, nullptr) : -1;
  f.nv_p = f.id_p >= 0 ? min(64, len - (pg0 + pp) * 64) : 0;
  const int id_o = c < np ? page_id(a, b, pg0 + c, nullptr) : -1;
  f.nv_o = id_o >= 0 ? min(64, len - (pg0 + c) * 64) : 64;
  f.full = f.nv_p == 64 && f.nv_o == 64;
  return f;
}

__device__ __forceinline__ uint32_t pack_bf162(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// One lane of the (converged) warp returns true.
__device__ __forceinline__ bool elect_one() {
  uint32_t is_leader;
  asm volatile("{\n\t.reg .pred p;\n\telect.sync _|p, 0xffffffff;\n\tselp.u32 %0, 1, 0, p;\n\t}" : "=r"(is_leader));
  return is_leader != 0;
}

// 16-byte copy global -> shared through L2; src_bytes = 0 writes 16 zero bytes.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
// Arrive on a local mbarrier once this thread's earlier cp.async copies have landed
// (the barrier's expected count includes this arrival).
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

__global__ void __launch_bounds__(kThreads, 1)
decode_pair_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tp,
                   const PairParams prm) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* sm =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* q_s = sm + kOffQ;
  unsigned char* p_s = sm + kOffP;
  unsigned char* buf_s = sm + kOffBuf;
  float* xch_m = reinterpret_cast<float*>(sm + kOffXch);   // [step parity][key half][TMEM lane]
  float* xch_l = xch_m + 512;                              // [key half][TMEM lane]
  PlanSmem* plan = reinterpret_cast<PlanSmem*>(sm + kOffPlan);
  Bars* bar = reinterpret_cast<Bars*>(sm + kOffBar);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sm + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + kOffMisc + 16);

  const DecodeArgs& a = prm.d;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t c = cluster_ctarank();
  const int w = blockIdx.x >> 1;
  const int row0 = blockIdx.y * 128;
  const long long lim = prm.spin_limit;
  int32_t* status = a.dev_status;

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar->kfull[s], 2);
      mbar_init(&bar->buf_lo[s], 1);
      mbar_init(&bar->buf_free[s], 1);
      mbar_init(&bar->vland[s], 32);
      mbar_init(&bar->vfull[s], 2);
      mbar_init(&bar->s_full[s], 1);
      mbar_init(&bar->s_empty[s], 16);
    }
    mbar_init(&bar->q_full, 2);
    mbar_init(&bar->qt_full, 16);
    mbar_init(&bar->q_empty, 1);
    mbar_init(&bar->p_full[0], 16);
    mbar_init(&bar->p_full[1], 16);
    mbar_init(&bar->p_empty[0], 1);
    mbar_init(&bar->p_empty[1], 1);
    mbar_init(&bar->o_free, 16);
    mbar_init(&bar->drain, 2);
    mbar_init(&bar->xm, 8);
    mbar_init(&bar->xl, 8);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch(&tq);
    tma_prefetch(&tp);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_holder, kTmemCols);
    tmem_relinquish_pair();
  }
  // setup above touches no input: the predecessor on the stream may still run
  grid_dependency_wait();
  // only now may the combine launch: its prologue reads seq_lens and W_UV,
  // whose producers (if any) ran before this kernel's wait returned
  allow_dependent_launch();
  build_plan(plan, a.seq_lens, a.batch, a.nq, a.max_pages, a.page_size, a.G, a.piece_cost,
             (blockIdx.x == 0 && blockIdx.y == 0) ? status : nullptr, a.kv_rank, a.kv_ranks);  // ends with __syncthreads
  tc_fence_before();
  cluster_sync();  // barriers and TMEM of both CTAs ready before any remote traffic
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  auto wwait = [&](uint64_t* b, uint32_t parity) -> bool {
    return __all_sync(0xffffffffu, mbar_wait(b, parity, abort_flag, status, lim));
  };

  if (warp == 0) {
    // ------------------------------------------------------------ query and step buffers (TMA)
    const uint32_t kfull0 = mapa(smem_u32(&bar->kfull[0]), 0);
    const uint32_t qfull0 = mapa(smem_u32(&bar->q_full), 0);
    const int oob_row = a.num_pages * 64;   // a box starting here lies outside the pool: zero fill
    const uint64_t stream_policy = l2_policy_evict_first();   // pages are read once per call
    StepCursor cur(plan, a.batch, w);
    Step st;
    int t = 0;
    while (!*abort_flag && cur.next(&st)) {
      if (st.first) {
        // the previous piece's score MMAs must be done with the query tile
        if (st.p > 0 && !wwait(&bar->q_empty, (st.p - 1) & 1)) break;
        if (lane == 0) {
          const int qrow = st.b * prm.rows_total + row0 + 64 * (int)c;
          mbar_arrive_expect_tx_cluster(qfull0, kQBytes);
          for (int i = 0; i < 5; ++i) tma_load_2d_pair(q_s + i * kBlockBytes, &tq, 256 + 64 * i, qrow, qfull0);
        }
      }
      const int u = t & 1;
      // the value MMAs of step t - 2 must be done with this buffer: the blocks
      // they read for page 0 (0, 1, 4, 5 and block 8, page 0's P) are free once
      // those MMAs are done, so their loads start before the page-1 MMAs complete
      int y = 0;
      if (lane == 0) {
        const int id = (int)c < st.np ? page_id(a, st.b, st.pg0 + (int)c, status) : -1;
        y = id >= 0 ? id * 64 : oob_row;
      }
      unsigned char* dst = buf_s + u * kBufBytes;
      if (t >= 2 && !wwait(&bar->buf_lo[u], ((t >> 1) - 1) & 1)) break;
      if (lane == 0) {
        mbar_arrive_expect_tx_cluster(kfull0 + 8 * u, kBufBytes);
        for (int k = 0; k < 5; ++k) {             // blocks 0, 1, 4, 5, 8
          const int blk = k == 4 ? 8 : (k & 1) + 4 * (k >> 1);
          tma_load_2d_pair_hint(dst + blk * kBlockBytes, &tp, 64 * blk, y, kfull0 + 8 * u, stream_policy);
        }
      }
      if (t >= 2 && !wwait(&bar->buf_free[u], ((t >> 1) - 1) & 1)) break;
      if (lane == 0)
        for (int k = 0; k < 4; ++k) {             // blocks 2, 3, 6, 7
          const int blk = 2 + (k & 1) + 4 * (k >> 1);
          tma_load_2d_pair_hint(dst + blk * kBlockBytes, &tp, 64 * blk, y, kfull0 + 8 * u, stream_policy);
        }
      ++t;
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ peer half of the value operand
    // Once a step's score MMAs are done, blocks 4j + 2(1-c) + e of its buffer (the
    // other half of the own page, no longer needed) receive the peer page's latent
    // columns 256j + 128c + 64e, e = 0, 1, read from L2 (the peer has just loaded
    // that page).  When both pages of the step are complete, four TMA boxes do it
    // and count their bytes on CTA 0's vfull directly.  Otherwise per-thread copies
    // zero the slots past the sequence's end, in the peer half and in the own half
    // (P = 0 does not cancel NaN in the product); they signal vland, and warp 3
    // hands the step on.
    const char* pool = reinterpret_cast<const char*>(a.pool);
    const uint32_t vfull0 = mapa(smem_u32(&bar->vfull[0]), 0);
    const uint64_t stream_policy = l2_policy_evict_first();
    StepCursor cur(plan, a.batch, w);
    Step st;
    int t = 0;
    uint32_t n_part = 0;   // partial steps so far (they alternate between the two vland barriers)
    while (!*abort_flag && cur.next(&st)) {
      const int u = t & 1;
      const int pp = 1 - (int)c;                                  // the peer's page of the step
      // page ids and lengths are read before the wait, off the critical path
      const PeerFetch f = peer_fetch(a, st.b, st.pg0, st.np, (int)c);
      if (!wwait(&bar->s_full[u], (t >> 1) & 1)) break;
      unsigned char* buf = buf_s + u * kBufBytes;
      if (f.full) {
        if (lane == 0) {
          mbar_arrive_expect_tx_cluster(vfull0 + 8 * u, 4 * kBlockBytes);
          for (int je = 0; je < 4; ++je) {
            const int j = je >> 1, e = je & 1;
            tma_load_2d_pair_hint(buf + (4 * j + 2 * pp + e) * kBlockBytes, &tp, 256 * j + 128 * (int)c + 64 * e,
                                  f.id_p * 64, vfull0 + 8 * u, stream_policy);
          }
        }
        __syncwarp();
        ++t;
        continue;
      }
      const char* src_p = pool + (size_t)(f.id_p >= 0 ? f.id_p : 0) * 64 * 1152;
      const uint32_t base = smem_u32(buf);
#pragma unroll 1
      for (int je = 0; je < 4; ++je) {
        const int j = je >> 1, e = je & 1;
        const uint32_t blk_p = base + (4 * j + 2 * pp + e) * kBlockBytes;
        const char* src = src_p + (256 * j + 128 * (int)c + 64 * e) * 2;
#pragma unroll 4
        for (int q = 0; q < 16; ++q) {
          const int idx = lane + 32 * q;                          // key = idx / 8, 16-byte piece = idx % 8
          const int key = idx >> 3, ch = idx & 7;
          const bool valid = key < f.nv_p;
          cp_async16(blk_p + key * 128 + ((ch ^ (key & 7)) << 4),
                     valid ? (const void*)(src + (size_t)key * 1152 + ch * 16) : (const void*)pool, valid ? 16u : 0u);
        }
        if (f.nv_o < 64) {
          const uint32_t blk_o = base + (4 * j + 2 * (int)c + e) * kBlockBytes;
          for (int idx = f.nv_o * 8 + lane; idx < 512; idx += 32)
            cp_async16(blk_o + (idx >> 3) * 128 + (((idx & 7) ^ ((idx >> 3) & 7)) << 4), pool, 0u);
        }
      }
      cp_async_arrive_noinc(&bar->vland[n_part & 1]);
      ++n_part;
      ++t;
    }
    cp_async_wait_all();
  } else if (warp == 3) {
    // ------------------------------------------------------------ hand a partial step's value operand on
    const uint32_t vfull0 = mapa(smem_u32(&bar->vfull[0]), 0);
    const uint64_t stream_policy = l2_policy_evict_first();
    StepCursor cur(plan, a.batch, w);
    Step st;
    int t = 0;
    uint32_t n_part = 0;
    while (cur.next(&st)) {
      const int u = t & 1;
      if (!peer_fetch(a, st.b, st.pg0, st.np, (int)c).full) {
        if (!wwait(&bar->vland[n_part & 1], (n_part >> 1) & 1)) break;
        ++n_part;
        fence_proxy_async_smem();           // the copies are read by the tensor core (async proxy)
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(vfull0 + 8 * u);
      }
      ++t;
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ score MMA issuer (CTA 0)
    // The score and the value MMAs are issued by two warps (1 and 12), so that
    // neither waits behind the other's issue loop (the MMA queue is shallow:
    // issuing stalls while the tensor core works through it), and each commit
    // tracks its own warp's MMAs only.  The whole warp runs the loop and waits;
    // one elected lane issues (an MMA issued from a lone lane under
    // data-dependent control flow costs several times its execution time).
    if (c == 0) {
      const uint32_t id_s = idesc_bf16_f32(128, 128, 0, 0);
      const uint32_t qa = smem_u32(q_s), ba = smem_u32(buf_s);
      StepCursor cur(plan, a.batch, w);
      Step st;
      int t = 0;
      while (cur.next(&st)) {
        if (st.first && (!wwait(&bar->q_full, st.p & 1) || !wwait(&bar->qt_full, st.p & 1))) break;
        if (t >= 2 && !wwait(&bar->s_empty[t & 1], ((t >> 1) - 1) & 1)) break;
        if (!wwait(&bar->kfull[t & 1], (t >> 1) & 1)) break;
        const uint32_t bu = ba + (t & 1) * kBufBytes;
        const uint32_t d = tmem + 64 * (t & 1);
        tc_fence_after();
        if (elect_one()) {
#pragma unroll
          for (int ks = 0; ks < 36; ++ks) {         // 16-column steps of the 576-wide dot product
            const uint64_t db = smem_desc(bu + (ks >> 2) * kBlockBytes + (ks & 3) * 32, 16, 1024, kSwizzle128);
            if (ks < 16) {
              mma_bf16_pair_ts(d, tmem + kTmemQ + 8 * ks, db, id_s, ks > 0 ? 1u : 0u);
            } else {
              const uint64_t da = smem_desc(qa + ((ks - 16) >> 2) * kBlockBytes + (ks & 3) * 32, 16, 1024,
                                            kSwizzle128);
              mma_bf16_pair(d, da, db, id_s, 1u);
            }
          }
          mma_commit_pair(&bar->s_full[t & 1]);
          if (st.last) mma_commit_pair(&bar->q_empty);
        }
        __syncwarp();
        ++t;
      }
      // drain: every MMA this warp issued has completed (and every commit before
      // this one has arrived) before TMEM and shared memory go away; the value
      // issuer commits to the same barrier
      if (elect_one()) mma_commit_pair(&bar->drain);
      __syncwarp();
      if (lane == 0) mbar_wait_drain(&bar->drain, 0, kDrainCycles + lim);
      __syncwarp();
    } else if (lane == 0) {
      // the leader's MMAs write this CTA's TMEM and its commits arrive here
      mbar_wait_drain(&bar->drain, 0, kDrainCycles + lim);
    }
  } else if (warp == 12) {
    // ------------------------------------------------------------ value MMA issuer (CTA 0)
    if (c == 0) {
      const uint32_t id_v = idesc_bf16_f32(128, 256, 0, 1);
      const uint32_t pa = smem_u32(p_s), ba = smem_u32(buf_s);
      StepCursor cur(plan, a.batch, w);
      Step st;
      int t = 0;
      while (cur.next(&st)) {
        // the previous piece's epilogue must have read O before the first value
        // MMA of this piece overwrites it
        if (st.first && st.p > 0 && !wwait(&bar->o_free, (st.p - 1) & 1)) break;
        if (!wwait(&bar->p_full[t & 1], (t >> 1) & 1)) break;
        if (!wwait(&bar->vfull[t & 1], (t >> 1) & 1)) break;
        const uint32_t bu = ba + (t & 1) * kBufBytes;
        tc_fence_after();
        if (elect_one()) {
#pragma unroll
          for (int pg = 0; pg < 2; ++pg)
#pragma unroll
            for (int j = 0; j < 2; ++j)
#pragma unroll
              for (int ks = 0; ks < 4; ++ks) {      // 16 keys of page pg per MMA
                // P of page 0 sits in the step buffer's rope block, free once the
                // scores are done; P of page 1 in P region [t & 1]
                const uint32_t pblk = pg == 0 ? bu + 8 * kBlockBytes : pa + (t & 1) * kBlockBytes;
                const uint64_t da = smem_desc(pblk + ks * 32, 16, 1024, kSwizzle128);
                const uint64_t db = smem_desc(bu + (4 * j + 2 * pg) * kBlockBytes + ks * 2048, kBlockBytes, 1024,
                                              kSwizzle128);
                mma_bf16_pair(tmem + kTmemO + 128 * j, da, db, id_v, (st.first && pg == 0 && ks == 0) ? 0u : 1u);
                // page 0's value blocks (0, 1, 4, 5) and its P (block 8) are done
                if (pg == 0 && j == 1 && ks == 3) mma_commit_pair(&bar->buf_lo[t & 1]);
              }
          mma_commit_pair(&bar->p_empty[t & 1]);
          mma_commit_pair(&bar->buf_free[t & 1]);
        }
        __syncwarp();
        ++t;
      }
      if (elect_one()) mma_commit_pair(&bar->drain);
      __syncwarp();
    }
  } else {
    // ------------------------------------------------------------ softmax warps
    // warps 4..11: warp w reads TMEM lane quarter w & 3 and key half kh of the
    // step's S (columns [32 kh, 32 kh + 32)); four threads share a row: its two
    // pages (lanes L and L ^ 64) times the two key halves
    const int quarter = warp & 3;
    const int kh = (warp - 4) >> 2;
    const int L = quarter * 32 + lane;                // this thread's TMEM lane
    const int r = L & 63, h = L >> 6;                 // row of this CTA, page of the step
    const int row = 64 * (int)c + r;                  // row of the tile
    const bool row_valid = row0 + row < prm.rows_total;
    const int qi = (row0 + row) / a.n_heads;          // query token of this row
    const uint32_t lane_off = uint32_t(quarter * 32) << 16;
    const uint32_t s_empty0 = mapa(smem_u32(&bar->s_empty[0]), 0);
    const uint32_t p_full0 = mapa(smem_u32(&bar->p_full[0]), 0);
    const uint32_t o_free0 = mapa(smem_u32(&bar->o_free), 0);
    const uint32_t qt_full0 = mapa(smem_u32(&bar->qt_full), 0);
    // latent columns [0,256) of this thread's query row into TMEM (both lanes of a
    // row hold it), for the first score MMAs of a piece
    auto load_query = [&](const Step& s) {
      const bool valid = row0 + row < prm.rows_total;   // rows past the tile's end read nothing
      const uint16_t* src = a.q_lat + ((size_t)s.b * prm.rows_total + row0 + row) * 576;
#pragma unroll 1
      for (int cc = 2 * kh; cc < 2 * kh + 2; ++cc) {   // half of the chunks each
        uint32_t v[32];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint4 x = valid ? ldg_stream(src + 64 * cc + 8 * i) : make_uint4(0, 0, 0, 0);
          v[4 * i] = x.x; v[4 * i + 1] = x.y; v[4 * i + 2] = x.z; v[4 * i + 3] = x.w;
        }
        tmem_st32_bits(tmem + lane_off + kTmemQ + 32 * cc, v);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(qt_full0);
    };
    // a page that the page table maps outside the pool is masked whole (its data
    // were zero-filled); the page id and the sequence length of a step are read
    // one step ahead, so that no load is outstanding at the arrives below (a
    // release would wait for it)
    auto page_ok = [&](const Step& s) { return h < s.np && page_id(a, s.b, s.pg0 + h, nullptr) >= 0; };
    StepCursor cur(plan, a.batch, w);
    Step st, nx;
    bool has = cur.next(&st);
    if (has) load_query(st);
    bool pg_ok = has && page_ok(st);
    int len = has ? a.seq_lens[st.b] : 0;
    float m_used = -INFINITY, l = 0.f;
    int vis = 0;    // last key index this row may see
    int t = 0;
    while (has) {
      const bool has_next = cur.next(&nx);
      if (st.first) {
        m_used = -INFINITY;
        l = 0.f;
        vis = min(len - 1, len - a.nq + qi);
      }
      if (!wwait(&bar->s_full[t & 1], (t >> 1) & 1)) break;
      tc_fence_after();
      float s[32];
      tmem_ld32(tmem + lane_off + 64 * (t & 1) + 32 * kh, s);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote_relaxed(s_empty0 + 8 * (t & 1));   // the TMEM reads are complete
      // keys [0, lim_k] of page h of the step are visible to this row, counted from
      // this thread's first key (key 32 kh of the page)
      const int lim_k = (row_valid && pg_ok) ? min(vis - (st.pg0 + h) * 64, 63) - 32 * kh : -1;
      float mx;
      {
        if (lim_k < 31) {                                // keys past the visible end
#pragma unroll
          for (int i = 0; i < 32; ++i) s[i] = i <= lim_k ? s[i] : -INFINITY;
        }
        float tt[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) tt[i] = -INFINITY;
#pragma unroll
        for (int i = 0; i < 32; ++i) tt[i & 3] = fmaxf(tt[i & 3], s[i]);
        // in log2 units: the scale is positive, so the max of the scaled scores is
        // the scaled max (rounding is monotonic); -inf stays -inf
        mx = fmaxf(fmaxf(tt[0], tt[1]), fmaxf(tt[2], tt[3])) * prm.scale_log2;
      }
      // the four threads of a row (two pages, lanes L and L ^ 64, times two key
      // halves) agree on the step's row max (a bounded mbarrier, not a named
      // barrier: a warp that gives up after a time-out must not leave the others
      // waiting)
      float* xm_s = xch_m + (t & 1) * 256;
      xm_s[kh * 128 + L] = mx;
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar->xm);
      if (!wwait(&bar->xm, t & 1)) break;
      mx = fmaxf(fmaxf(xm_s[L], xm_s[L ^ 64]), fmaxf(xm_s[128 + L], xm_s[128 + (L ^ 64)]));
      const float m_new = fmaxf(m_used, mx);
      const bool grow = m_new > m_used + kRescaleThreshold;
      // P is double-buffered: its blocks for this step were last read by the value
      // MMAs of step t - 2, done before this step's buffer was loaded.  Only a
      // rescale of O waits for the value MMAs of the previous step.  The two warps
      // of a lane quarter hold the same rows and decide alike; each rescales its
      // half of the row's O columns.
      if (__any_sync(0xffffffffu, grow && m_used != -INFINITY)) {
        if (!wwait(&bar->p_empty[(t - 1) & 1], ((t - 1) >> 1) & 1)) break;
        const float alpha = (grow && m_used != -INFINITY) ? ex2(m_used - m_new) : 1.f;
        tc_fence_after();
#pragma unroll 1
        for (int cc = 128 * kh; cc < 128 * kh + 128; cc += 32) {
          float o[32];
          tmem_ld32(tmem + lane_off + kTmemO + cc, o);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] *= alpha;
          tmem_st32(tmem + lane_off + kTmemO + cc, o);
        }
        tmem_wait_st();
        l *= alpha;
      }
      if (grow) m_used = m_new;
      const float m_ref = (m_used == -INFINITY) ? 0.f : m_used;
      float ps[4] = {0.f, 0.f, 0.f, 0.f};
      unsigned char* prow = (h == 0 ? buf_s + (t & 1) * kBufBytes + 8 * kBlockBytes : p_s + (t & 1) * kBlockBytes) +
                            r * 128;                   // P block h: the keys of page h
#pragma unroll
      for (int cq = 0; cq < 4; ++cq) {                   // 16-byte chunks 4 kh .. 4 kh + 3 of the row
        const int ch = 4 * kh + cq;
        uint32_t pk[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int i = 8 * cq + 2 * e;
          const float p0 = ex2(fmaf(s[i], prm.scale_log2, -m_ref));       // ex2(-inf) = 0
          const float p1 = ex2(fmaf(s[i + 1], prm.scale_log2, -m_ref));
          ps[e] += p0 + p1;
          pk[e] = pack_bf162(p0, p1);
        }
        *reinterpret_cast<uint4*>(prow + ((ch ^ (r & 7)) << 4)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      }
      l += (ps[0] + ps[1]) + (ps[2] + ps[3]);
      fence_proxy_async_smem();                          // P -> tensor core (async proxy)
      tc_fence_before();                                 // O rescale -> MMA
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(p_full0 + 8 * (t & 1));
      // the next step's loads, issued after the release above
      const bool pg_ok_next = has_next && page_ok(nx);
      const int len_next = has_next ? a.seq_lens[nx.b] : 0;

      if (st.last) {
        // the score MMAs of this piece are done (its last S was read above): the
        // next piece's query may go into TMEM before this piece's epilogue
        if (has_next) load_query(nx);
        // epilogue: O / l and lse of the piece; l summed over the row's four
        // threads, in the same order in each of them
        xch_l[kh * 128 + L] = l;
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar->xl);
        if (!wwait(&bar->xl, st.p & 1)) break;
        const int l0 = L & 63;
        const float lt = (xch_l[l0] + xch_l[128 + l0]) + (xch_l[64 + l0] + xch_l[192 + l0]);
        // O is final once the value MMAs of this step are done (their commit also
        // covers every earlier MMA)
        if (!wwait(&bar->p_empty[t & 1], (t >> 1) & 1)) break;
        tc_fence_after();
        const float inv_l = lt > 0.f ? 1.f / lt : 0.f;
        float* dst = a.part_o + ((size_t)st.id * prm.rows_total + row0 + row) * a.d_c + 128 * h;
#pragma unroll 1
        for (int cc = 128 * kh; cc < 128 * kh + 128; cc += 32) {
          float o[32];
          tmem_ld32(tmem + lane_off + kTmemO + cc, o);
          tmem_wait_ld();
          if (row_valid) {
            float* dd = dst + 256 * (cc >> 7) + (cc & 127);
#pragma unroll
            for (int i = 0; i < 32; i += 4)
              *reinterpret_cast<float4*>(dd + i) =
                  make_float4(o[i] * inv_l, o[i + 1] * inv_l, o[i + 2] * inv_l, o[i + 3] * inv_l);
          }
        }
        if (row_valid && h == 0 && kh == 0)
          a.part_lse[(size_t)st.id * prm.rows_total + row0 + row] =
              lt > 0.f ? (m_used + log2f(lt)) * 0.6931471805599453f : -INFINITY;
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_remote_relaxed(o_free0);   // the TMEM reads are complete
      }
      st = nx;
      has = has_next;
      pg_ok = pg_ok_next;
      len = len_next;
      ++t;
    }
  }

  // ------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (*abort_flag) {
    // after a time-out, copies this CTA issued may still be in flight (their
    // completion is counted in CTA 0): give them time to land before exiting
    const long long t0 = clock64();
    while (clock64() - t0 < 200000) __nanosleep(1000);
  }
  cluster_sync();  // the peer no longer touches this CTA's shared memory or TMEM
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kTmemCols);
  }
}

}  // namespace

bool decode_pair_supported(int d_c, int d_rope, int page_size) { return d_c == 512 && d_rope == 64 && page_size == 64; }

int decode_pair_workers(int sms, int rows_total) {
  const int tiles = (rows_total + 127) / 128;
  const int g = (sms / 2) / tiles;
  return g < 1 ? 1 : g;
}

cudaError_t launch_decode_split_pair(const DecodeArgs& a, long long spin_limit, cudaStream_t stream) {
  const int rows_total = a.nq * a.n_heads;
  CUtensorMap tq, tp;
  const uint64_t qrows = (uint64_t)a.batch * rows_total;
  const uint64_t prows = (uint64_t)a.num_pages * 64;
  if (!encode_rows576(&tq, a.q_lat, qrows, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_rows576(&tp, a.pool, prows, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  PairParams prm;
  prm.d = a;
  prm.rows_total = rows_total;
  prm.scale_log2 = a.scale * 1.4426950408889634f;
  prm.spin_limit = spin_limit;
  cudaError_t e = cudaFuncSetAttribute(decode_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * a.G, (rows_total + 127) / 128, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1] = pdl_attribute();
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  e = cudaLaunchKernelEx(&cfg, decode_pair_kernel, tq, tp, prm);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace mla
