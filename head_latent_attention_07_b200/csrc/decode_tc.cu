// Split-KV latent attention on the 5th-generation tensor cores (tcgen05, TMEM, TMA).
//
// Shape: d_c = 512, d_rope = 64 (576-wide cache rows), 64-token pages, up to 128
// query rows (query token, head) per tile.
//
// A CTA pair (cluster of 2) works on one (worker, row tile).  CTA c owns latent
// columns [256c, 256c + 256) and RoPE columns [512 + 32c, 512 + 32c + 32) of
// every cache row and of the query tile, so each page is read from HBM once per
// pair, half by each CTA.  Per page (64 tokens):
//   GEMM1   S_c[128 x 64] = Q_c[128 x 288] . K_c[64 x 288]^T: partial scores over
//           this CTA's columns (latent part of Q_c in TMEM, RoPE part and the page
//           in shared memory)
//   swap    CTA c owns the softmax of keys [32c, 32c + 32) of every row: it sends
//           the peer the partial scores of the peer's keys (fp32, log2 units) and
//           adds the peer's partials of its own keys to its fp32 ones
//   softmax the two CTAs agree on each row's running max (one float per row each
//           way); each computes P (bf16) for its 32 keys and writes it into both
//           CTAs' P tiles
//   GEMM2   O_c[128 x 256] += P[128 x 64] . C_c[64 x 256]  (P and page in shared
//           memory, O in TMEM)
// The running max is only moved (and O rescaled in TMEM, by both CTAs alike) when
// it grows by more than 2^8; otherwise P is taken relative to the stale max.
// Each CTA keeps the row sums of its own keys; the two halves are added at the
// end of every piece, and each CTA normalises its own 256 columns of O.
// TMEM: O columns [0, 256), S buffers [256, 320) and [320, 384), Q latent
// (bf16 pairs) [384, 512).
//
// Warp roles (320 threads): warp 0 lane 0 issues TMA loads (RoPE part of the
// query tile once per piece, pages into a 4-stage ring), warp 1 owns TMEM and lane 0 issues the MMAs, warps 2..5 (one per TMEM
// lane quarter, one query row per thread) load the query tile's latent part into
// TMEM and send the peer its partial scores, and warps 6..9 (same layout) run the
// softmax and the epilogue.
// Every mbarrier wait is bounded: on time-out the kernel records MLA_ERR_TIMEOUT,
// stops its loops, drains its own copies and MMAs and frees TMEM.
#include <cuda.h>
#include <cuda_fp16.h>

#include <mutex>

#include "common.cuh"
#include "decode.h"
#include "plan.cuh"
#include "sm100.cuh"

namespace mla {

namespace {

using namespace sm100;

constexpr int kThreads = 320;  // producer, MMA, 4 sender warps, 4 softmax warps
constexpr int kStages = 4;
constexpr int kQrBytes = 128 * 64;            // RoPE block of the query tile [128 x 32] (64-byte swizzle)
constexpr int kPageBytes = 4 * 8192 + 4096;   // 4 latent blocks [64 x 64] + RoPE block [64 x 32]
constexpr int kXBytes = 128 * 128;            // received partial scores: [128 rows x 32 keys] fp32
constexpr int kPBytes = 128 * 128;            // P tile [128 rows x 64 keys] bf16, 128-byte swizzle
constexpr int kPTiles = 2;                    // P of pages k, k + 1 in flight
constexpr int kOffQr = 0;
constexpr int kOffPg = kOffQr + kQrBytes;
constexpr int kOffX = kOffPg + kStages * kPageBytes;
constexpr int kOffP = kOffX + 2 * kXBytes;
constexpr int kOffM = kOffP + kPTiles * kPBytes;  // received row maxima [2][128], row sums [128] (fp32)
constexpr int kOffPlan = kOffM + 3 * 128 * 4;
constexpr int kOffBar = kOffPlan + ((int(sizeof(PlanSmem)) + 15) & ~15);
constexpr int kNumBars = 32;
constexpr int kOffMisc = kOffBar + kNumBars * 8;       // TMEM base, abort flag, page metadata
constexpr int kSmemBytes = kOffMisc + 64 + 1024;       // + 1 KB alignment slack
constexpr float kRescaleThreshold = 8.0f;     // log2 units: rescale when the max grows by > 2^8
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemS = 256;              // S buffers: columns [256, 320) and [320, 384)
constexpr uint32_t kTmemQ = 384;              // Q latent, 256 bf16 per row: columns [384, 512)

static_assert(kSmemBytes <= 232448, "shared memory budget");
static_assert(kOffPg % 1024 == 0 && kPageBytes % 1024 == 0 && kOffP % 1024 == 0, "swizzle alignment");

struct TcParams {
  DecodeArgs d;
  int rows_total;   // nq * H
  float scale_log2; // softmax scale * log2(e)
  long long spin_limit;
};

struct Bars {
  uint64_t q_full, q_empty;
  uint64_t pg_full[kStages], pg_empty[kStages];
  uint64_t s_full[2], s_empty[2];
  uint64_t x_full[2], x_free[2];   // partial scores from the peer / the peer's slot is free
  uint64_t m_full[2];              // the peer's row maxima of a page
  uint64_t p_full[kPTiles], p_free[kPTiles];  // P tile complete (own + peer half) / the peer's P tile is free
  uint64_t o_done[kPTiles];        // this CTA's value MMAs of the page that used the tile are done
  uint64_t l_full, o_free, drain;
};
static_assert(sizeof(Bars) <= kNumBars * 8, "barrier area");

// Walks the pages of worker w: jj counts pages across pieces, p counts pieces.
struct PageCursor {
  PieceIter it;
  Piece pc;
  int pg = 0, jj = -1, p = -1;
  bool in_piece = false;
  __device__ PageCursor(const PlanSmem* ps, int batch, int w) : it(ps, batch, w) {}
  __device__ bool next() {
    if (in_piece && pg + 1 < pc.pg_end) {
      ++pg;
      ++jj;
      return true;
    }
    if (!it.next(&pc)) {
      in_piece = false;
      return false;
    }
    in_piece = true;
    pg = pc.pg_begin;
    ++jj;
    ++p;
    return true;
  }
  __device__ bool first() const { return pg == pc.pg_begin; }
  __device__ bool last() const { return pg == pc.pg_end - 1; }
};

// One lane of the (converged) warp returns true.
__device__ __forceinline__ bool elect_one() {
  uint32_t is_leader;
  asm volatile("{\n\t.reg .pred p;\n\telect.sync _|p, 0xffffffff;\n\tselp.u32 %0, 1, 0, p;\n\t}" : "=r"(is_leader));
  return is_leader != 0;
}

__device__ __forceinline__ uint32_t pack_bf162(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}


__global__ void __launch_bounds__(kThreads, 1)
decode_split_tc_kernel(const __grid_constant__ CUtensorMap tq64, const __grid_constant__ CUtensorMap tp128,
                       const __grid_constant__ CUtensorMap tp64, const TcParams prm) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* sm =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* qr_s = sm + kOffQr;
  unsigned char* pg_s = sm + kOffPg;
  unsigned char* x_s = sm + kOffX;
  unsigned char* p_s = sm + kOffP;
  float* m_recv = reinterpret_cast<float*>(sm + kOffM);         // [2][128]
  float* l_recv = m_recv + 256;                                 // [128]
  PlanSmem* plan = reinterpret_cast<PlanSmem*>(sm + kOffPlan);
  Bars* bar = reinterpret_cast<Bars*>(sm + kOffBar);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sm + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + kOffMisc + 16);
  int* stage_nvalid = reinterpret_cast<int*>(sm + kOffMisc + 32);   // [kStages] valid keys of the page

  const DecodeArgs& a = prm.d;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t c = cluster_ctarank();
  const uint32_t peer = c ^ 1u;
  const int w = blockIdx.x >> 1;
  const int row0 = blockIdx.y * 128;
  const int rows_valid = min(128, prm.rows_total - row0);
  const long long lim = prm.spin_limit;
  int32_t* status = a.dev_status;

  if (threadIdx.x == 0) {
    mbar_init(&bar->q_full, 5);        // 4 sender warps (latent part) + producer (RoPE part, bytes)
    mbar_init(&bar->q_empty, 1);
    for (int s = 0; s < kStages; ++s) { mbar_init(&bar->pg_full[s], 1); mbar_init(&bar->pg_empty[s], 1); }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar->s_full[s], 1);
      mbar_init(&bar->s_empty[s], 8);  // 4 sender warps + 4 softmax warps read S
      mbar_init(&bar->x_full[s], 1);   // local softmax leader's expect-bytes arrival; the peer's stores carry the bytes
      mbar_init(&bar->x_free[s], 4);   // the peer's 4 softmax warps have read their slot
      mbar_init(&bar->m_full[s], 1);
    }
    for (int s = 0; s < kPTiles; ++s) {
      mbar_init(&bar->p_full[s], 4);   // 4 local softmax warps (one also expects the peer's bytes)
      mbar_init(&bar->p_free[s], 1);   // the peer's value MMA of the page has read its P tile
      mbar_init(&bar->o_done[s], 1);
    }
    mbar_init(&bar->l_full, 1);
    mbar_init(&bar->o_free, 4);
    mbar_init(&bar->drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch(&tq64); tma_prefetch(&tp128); tma_prefetch(&tp64);
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, kTmemCols);
    tmem_relinquish();
  }
  // setup above touches no input: the predecessor on the stream may still run
  grid_dependency_wait();
  // only now may the combine launch: its prologue reads seq_lens and W_UV,
  // whose producers (if any) ran before this kernel's wait returned
  allow_dependent_launch();
  build_plan(plan, a.seq_lens, a.batch, a.nq, a.max_pages, a.page_size, a.G,
             (blockIdx.x == 0 && blockIdx.y == 0) ? status : nullptr, a.kv_rank, a.kv_ranks);  // ends with __syncthreads
  tc_fence_before();
  cluster_sync();  // barriers of both CTAs initialised before any remote traffic
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      // No L2 prefetch ahead of the ring: measured on this kernel and on a bare
      // TMA stream of the same pages, prefetching slowed both (the prefetched
      // lines compete with the ring's own loads and are partly evicted first).
      PageCursor cu(plan, a.batch, w);
      int issued[kStages] = {0, 0, 0, 0}, issued_q = 0;
      bool more = cu.next();
      int id_next = more ? a.page_table[(size_t)cu.pc.b * a.max_pages + cu.pg] : 0;
      int len_next = more ? a.seq_lens[cu.pc.b] : 0;
      while (more && !*abort_flag) {
        const int jj = cu.jj;
        int id = id_next;
        const int nvalid_raw = min(64, len_next - cu.pg * 64);
        if (cu.first()) {
          if (cu.p > 0 && !mbar_wait(&bar->q_empty, (cu.p - 1) & 1, abort_flag, status, lim)) break;
          const int qrow = cu.pc.b * prm.rows_total + row0;
          mbar_arrive_expect_tx(&bar->q_full, kQrBytes);
          tma_load_2d(qr_s, &tq64, 512 + 32 * c, qrow, &bar->q_full);
          ++issued_q;
        }
        const int st = jj % kStages;
        more = cu.next();
        // the next page id is read while this stage drains
        if (more) {
          id_next = a.page_table[(size_t)cu.pc.b * a.max_pages + cu.pg];
          len_next = a.seq_lens[cu.pc.b];
        }
        if (jj >= kStages && !mbar_wait(&bar->pg_empty[st], ((jj / kStages) - 1) & 1, abort_flag, status, lim)) break;
        const bool page_ok = id >= 0 && id < a.num_pages;
        if (!page_ok) {
          record_status(status, MLA_ERR_RANGE);
          id = 0;  // loaded but never used: all its keys are masked and its rows zeroed
        }
        stage_nvalid[st] = page_ok ? nvalid_raw : 0;  // published by the arrive below
        unsigned char* dst = pg_s + st * kPageBytes;
        mbar_arrive_expect_tx(&bar->pg_full[st], kPageBytes);
        for (int i = 0; i < 4; ++i) tma_load_2d(dst + i * 8192, &tp128, c * 256 + 64 * i, id * 64, &bar->pg_full[st]);
        tma_load_2d(dst + 32768, &tp64, 512 + 32 * c, id * 64, &bar->pg_full[st]);
        ++issued[st];
      }
      if (*abort_flag) {
        // copies still in flight must land before this CTA's shared memory is released
        for (int s = 0; s < kStages; ++s)
          if (issued[s] > 0) mbar_wait_drain(&bar->pg_full[s], (issued[s] - 1) & 1, lim);
        if (issued_q > 0) mbar_wait_drain(&bar->q_full, (issued_q - 1) & 1, lim);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // Two in-order queues, each issued as soon as its inputs are ready: GEMM1
    // (scores, up to two pages ahead: S is double-buffered) and GEMM2 (values,
    // checked first).  The whole warp runs the loop: lane 0 tests the barriers and
    // walks the pages, the other lanes follow its decision word (broadcast by
    // shuffle), so that the MMA operands stay warp-uniform, and one elected lane
    // issues.  (Issued from a lone lane under data-dependent control flow, each MMA
    // cost several times its execution time on B200.)
    {
      constexpr uint32_t kGo1 = 1, kGo2 = 2, kFirst2 = 4, kLast1 = 8, kStop = 16;
      const uint32_t id1 = idesc_bf16_f32(128, 64, 0, 0);
      const uint32_t id2 = idesc_bf16_f32(128, 256, 0, 1);
      const uint32_t qra = smem_u32(qr_s);
      PageCursor g1(plan, a.batch, w), g2(plan, a.batch, w);
      bool has1 = false, has2 = false;
      if (lane == 0) {
        has1 = g1.next();
        has2 = g2.next();
      }
      bool q_ok = false;       // query tile of g1's piece is resident (lane 0)
      int jj1 = 0, jj2 = 0;    // pages issued by the two queues (all lanes)
      long long t_last = clock64();
      while (true) {
        uint32_t word = 0;
        if (lane == 0) {
          if (!has1 && !has2) {
            word = kStop;
          } else {
            if (has2 && (!has1 || g2.jj < g1.jj)) {
              const bool first = g2.first();
              if ((!(first && g2.p > 0) || mbar_test(&bar->o_free, (g2.p - 1) & 1)) &&
                  mbar_test(&bar->p_full[g2.jj % kPTiles], (g2.jj / kPTiles) & 1))
                word |= kGo2 | (first ? kFirst2 : 0);
            }
            if (has1) {
              const int jj = g1.jj;
              if (g1.first() && !q_ok) q_ok = mbar_test(&bar->q_full, g1.p & 1);
              if ((!g1.first() || q_ok) && (jj < 2 || mbar_test(&bar->s_empty[jj & 1], ((jj >> 1) - 1) & 1)) &&
                  mbar_test(&bar->pg_full[jj % kStages], (jj / kStages) & 1))
                word |= kGo1 | (g1.last() ? kLast1 : 0);
            }
            if (word & (kGo1 | kGo2)) {
              t_last = clock64();
            } else if (*abort_flag) {
              word = kStop;
            } else if (clock64() - t_last > lim) {
              record_status(status, MLA_ERR_TIMEOUT);
              *abort_flag = 1;
              word = kStop;
            }
          }
        }
        word = __shfl_sync(0xffffffffu, word, 0);
        if (word & kStop) break;
        if (word & kGo2) {
          const uint32_t pa = smem_u32(p_s + (jj2 % kPTiles) * kPBytes);
          const uint32_t pb = smem_u32(pg_s + (jj2 % kStages) * kPageBytes);
          if (elect_one()) {
            fence_proxy_async_smem();  // P written by threads of both CTAs, read by the tensor core
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
              const uint64_t da = smem_desc(pa + ks * 32, 16, 1024, kSwizzle128);
              const uint64_t db = smem_desc(pb + ks * 2048, 8192, 1024, kSwizzle128);
              mma_bf16(tmem, da, db, id2, ((word & kFirst2) && ks == 0) ? 0u : 1u);
            }
            mma_commit(&bar->pg_empty[jj2 % kStages]);
            mma_commit(&bar->o_done[jj2 % kPTiles]);
            // this CTA's P tile has been read: the peer may write page jj2 + kPTiles's half
            mma_commit_mc(&bar->p_free[jj2 % kPTiles], uint16_t(1u << peer));
          }
          __syncwarp();
          if (lane == 0) has2 = g2.next();
          ++jj2;
        }
        if (word & kGo1) {
          const uint32_t pb = smem_u32(pg_s + (jj1 % kStages) * kPageBytes);
          const uint32_t ts = tmem + kTmemS + 64 * (jj1 & 1);
          if (elect_one()) {
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 16; ++ks) {          // latent part: A from TMEM
              const uint64_t db = smem_desc(pb + (ks >> 2) * 8192 + (ks & 3) * 32, 16, 1024, kSwizzle128);
              mma_bf16_ts(ts, tmem + kTmemQ + 8 * ks, db, id1, ks > 0 ? 1u : 0u);
            }
#pragma unroll
            for (int ks = 0; ks < 2; ++ks) {           // RoPE part: A from shared memory
              const uint64_t da = smem_desc(qra + ks * 32, 16, 512, kSwizzle64);
              const uint64_t db = smem_desc(pb + 32768 + ks * 32, 16, 512, kSwizzle64);
              mma_bf16(ts, da, db, id1, 1u);
            }
            mma_commit(&bar->s_full[jj1 & 1]);
            if (word & kLast1) mma_commit(&bar->q_empty);
          }
          __syncwarp();
          if (lane == 0) {
            if (word & kLast1) q_ok = false;
            has1 = g1.next();
          }
          ++jj1;
        }
      }
      // drain: every MMA issued above has completed before TMEM / smem go away
      if (elect_one()) mma_commit(&bar->drain);
      __syncwarp();
      if (lane == 0) {
        mbar_wait_drain(&bar->drain, 0, lim);
        // the peer's value MMAs of the last kPTiles pages release this CTA's P tiles
        // by a multicast arrive that nothing else waits for: let it land
        const long long lim_drain = *abort_flag ? (1ll << 20) : lim;
        const int last2 = jj2 - 1;
        for (int jj = max(0, last2 - (kPTiles - 1)); jj <= last2; ++jj)
          mbar_wait_drain(&bar->p_free[jj % kPTiles], (jj / kPTiles) & 1, lim_drain);
      }
      __syncwarp();
    }
  } else if (warp < 6) {
    // ------------------------------------------------------------ sender warps
    // Per piece: the latent part of this CTA's query columns into TMEM.  Per
    // page: the partial scores of the peer's keys out of TMEM, scaled to log2
    // units, rounded to fp16 and stored into the peer's receive slot (k & 1).
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_off = uint32_t(quarter * 32) << 16;
    const uint32_t x_peer = mapa(smem_u32(x_s), peer);
    const uint32_t xfull_peer = mapa(smem_u32(&bar->x_full[0]), peer);
    const uint32_t sw = uint32_t(r & 7);               // chunk swizzle of row r in a receive slot
    auto wwait = [&](uint64_t* b, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(b, parity, abort_flag, status, lim));
    };
    PageCursor ca(plan, a.batch, w);
    int last_jj = -1;
    while (ca.next()) {
      const int jj = ca.jj;
      const int slot = jj & 1;
      if (ca.first()) {
        // the previous piece's score MMAs are done with TMEM's query columns
        if (ca.p > 0 && !wwait(&bar->q_empty, (ca.p - 1) & 1)) break;
        const uint16_t* qsrc = a.q_lat + ((size_t)ca.pc.b * prm.rows_total + row0 + r) * 576 + 256 * c;
#pragma unroll 1
        for (int cc = 0; cc < 4; ++cc) {                // 64 bf16 = 32 TMEM columns per chunk
          uint32_t v[32];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const uint4 u = r < rows_valid ? ldg_stream(qsrc + 64 * cc + 8 * i) : make_uint4(0, 0, 0, 0);
            v[4 * i] = u.x; v[4 * i + 1] = u.y; v[4 * i + 2] = u.z; v[4 * i + 3] = u.w;
          }
          tmem_st32_bits(tmem + lane_off + kTmemQ + 32 * cc, v);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar->q_full);
      }
      if (!wwait(&bar->s_full[slot], (jj >> 1) & 1)) break;
      tc_fence_after();
      float sv[32];
      tmem_ld32(tmem + kTmemS + 64 * slot + lane_off + 32 * peer, sv);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar->s_empty[slot]);
      // fp32 in log2 units: a half of the dot product can be large while the whole
      // score is not (opposite halves), and only fp32 keeps the sum's absolute error
      // small enough for the softmax weights
      uint32_t h[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) h[i] = __float_as_uint(sv[i] * prm.scale_log2);
      // the peer's receive slot is free once its softmax warps have read page jj - 2
      if (jj >= 2 && !wwait(&bar->x_free[slot], ((jj >> 1) - 1) & 1)) break;
      const uint32_t dst = x_peer + slot * kXBytes + r * 128;
      const uint32_t rbar = xfull_peer + slot * 8;
#pragma unroll
      for (int k4 = 0; k4 < 8; ++k4)
        st_async_v4(dst + ((k4 ^ sw) << 4), make_uint4(h[4 * k4], h[4 * k4 + 1], h[4 * k4 + 2], h[4 * k4 + 3]),
                    rbar);
      last_jj = jj;
    }
    // the peer's softmax warps release the last two slots after this loop ends:
    // their arrivals must land before this CTA's shared memory is released
    if (warp == 2 && lane == 0) {
      const long long lim_drain = *abort_flag ? (1ll << 20) : lim;
      for (int jj = max(0, last_jj - 1); jj <= last_jj; ++jj)
        mbar_wait_drain(&bar->x_free[jj & 1], (jj >> 1) & 1, lim_drain);
    }
  } else {
    // ------------------------------------------------------------ softmax warps
    // B(k), one query row per thread, this CTA's 32 keys of the page:
    //   S = own + peer: this CTA's fp32 partial (scaled) plus the peer's fp16 one,
    //   masked; the row max is agreed with the peer (both take the max of the two
    //   halves), P(k) (bf16) goes into both CTAs' P tiles, O is rescaled when the
    //   max grew, epilogue (O / l, lse) at the end of each piece.
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;                 // query row within the tile = TMEM lane
    const uint32_t lane_off = uint32_t(quarter * 32) << 16;
    const bool row_valid = r < rows_valid;
    const int qi = (row0 + r) / a.n_heads;             // query token of this row
    const int ltid = threadIdx.x - 192;                // 0..127
    const uint32_t sw = uint32_t(r & 7);
    const uint32_t xfree_peer = mapa(smem_u32(&bar->x_free[0]), peer);
    const uint32_t mrecv_peer = mapa(smem_u32(m_recv), peer);
    const uint32_t mfull_peer = mapa(smem_u32(&bar->m_full[0]), peer);
    const uint32_t lrecv_peer = mapa(smem_u32(l_recv), peer);
    const uint32_t lfull_peer = mapa(smem_u32(&bar->l_full), peer);
    const uint32_t p_peer = mapa(smem_u32(p_s), peer);
    const uint32_t pfull_peer = mapa(smem_u32(&bar->p_full[0]), peer);
    const bool leader = warp == 6 && lane == 0;        // posts the expected byte counts
    auto wwait = [&](uint64_t* b, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(b, parity, abort_flag, status, lim));
    };

    PageCursor cb(plan, a.batch, w);
    float m_used = -INFINITY, l = 0.f;
    int vis_last = 0;
    bool ok = true;
    while (ok && cb.next()) {
      const int jj = cb.jj;
      const int slot = jj & 1;
      const int st = jj % kStages;
      if (cb.first()) {
        m_used = -INFINITY;
        l = 0.f;
        vis_last = a.seq_lens[cb.pc.b] - a.nq + qi;    // last key index this row may see
      }
      if (!wwait(&bar->s_full[slot], (jj >> 1) & 1)) { ok = false; break; }
      tc_fence_after();
      float s[32];
      tmem_ld32(tmem + kTmemS + 64 * slot + lane_off + 32 * c, s);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar->s_empty[slot]);
      // the producer published the page's valid key count before its copy started
      mbar_try_wait(&bar->pg_full[st], (jj / kStages) & 1);  // complete already: acquire only
      const int nvalid = stage_nvalid[st];
      // keys 32c + [0, lim_h] are visible to this row
      const int lim_h = (row_valid ? min(nvalid - 1, vis_last - cb.pg * 64) : -1) - 32 * (int)c;
      // the peer's partial scores of this CTA's keys; the expected byte count is
      // posted by the consumer, once the slot's previous phase has completed
      if (leader) mbar_arrive_expect_tx(&bar->x_full[slot], kXBytes);
      if (!wwait(&bar->x_full[slot], (jj >> 1) & 1)) { ok = false; break; }
      const unsigned char* xrow = x_s + slot * kXBytes + r * 128;
#pragma unroll
      for (int k4 = 0; k4 < 8; ++k4) {                 // whole scores in log2 units
        const float4 v = *reinterpret_cast<const float4*>(xrow + ((k4 ^ sw) << 4));
        s[4 * k4] = fmaf(s[4 * k4], prm.scale_log2, v.x);
        s[4 * k4 + 1] = fmaf(s[4 * k4 + 1], prm.scale_log2, v.y);
        s[4 * k4 + 2] = fmaf(s[4 * k4 + 2], prm.scale_log2, v.z);
        s[4 * k4 + 3] = fmaf(s[4 * k4 + 3], prm.scale_log2, v.w);
      }
      // the peer may refill this slot: the loads above have returned (their values
      // are consumed), so the arrive needs no release ordering
      __syncwarp();
      if (lane == 0) mbar_arrive_remote_relaxed(xfree_peer + slot * 8);
      if (lim_h < 31) {                                // masked keys: past the length or causal
#pragma unroll
        for (int i = 0; i < 32; ++i) s[i] = (i <= lim_h) ? s[i] : -INFINITY;
      }
      float mx;
      {
        float t[8];                                    // tree reduction: short dependency chain
#pragma unroll
        for (int i = 0; i < 8; ++i) t[i] = fmaxf(fmaxf(s[i], s[i + 8]), fmaxf(s[i + 16], s[i + 24]));
#pragma unroll
        for (int n = 4; n > 0; n >>= 1)
#pragma unroll
          for (int i = 0; i < n; ++i) t[i] = fmaxf(t[i], t[i + n]);
        mx = t[0];
      }
      // swap the row maxima of the two key halves with the peer
      if (leader) mbar_arrive_expect_tx(&bar->m_full[slot], 128 * 4);
      st_async_b32(mrecv_peer + (slot * 128 + r) * 4, __float_as_uint(mx), mfull_peer + slot * 8);
      if (!wwait(&bar->m_full[slot], (jj >> 1) & 1)) { ok = false; break; }
      mx = fmaxf(mx, m_recv[slot * 128 + r]);          // both CTAs now hold the same row max

      // lazy running max: rescale O and l only when the max grows by more than 2^8
      const float m_new = fmaxf(m_used, mx);
      const bool grow = m_new > m_used + kRescaleThreshold;
      if (__any_sync(0xffffffffu, grow && !cb.first() && m_used != -INFINITY)) {
        const float alpha = (grow && m_used != -INFINITY) ? ex2(m_used - m_new) : 1.f;
        const int jp = jj - 1;  // O must hold every earlier page of this piece
        if (!wwait(&bar->o_done[jp % kPTiles], (jp / kPTiles) & 1)) { ok = false; break; }
        tc_fence_after();
#pragma unroll 1
        for (int cc = 0; cc < 256; cc += 32) {
          float o[32];
          tmem_ld32(tmem + lane_off + cc, o);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] *= alpha;
          tmem_st32(tmem + lane_off + cc, o);
        }
        tmem_wait_st();
        l *= alpha;
      }
      if (grow) m_used = m_new;
      const float m_ref = (m_used == -INFINITY) ? 0.f : m_used;
      uint32_t pk[16];
      float ps[4];                                     // 4 partial sums: short dependency chains
#pragma unroll
      for (int i = 0; i < 4; ++i) ps[i] = 0.f;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float p0 = ex2(s[2 * i] - m_ref);         // ex2(-inf) = 0
        const float p1 = ex2(s[2 * i + 1] - m_ref);
        ps[i & 3] += p0 + p1;
        pk[i] = pack_bf162(p0, p1);
      }
      l += (ps[0] + ps[1]) + (ps[2] + ps[3]);
      // P(k) -> P tile (k mod 3) of both CTAs, keys [32c, 32c + 32) of row r, once
      // the value MMAs of page k - 3 (own and peer) have read those tiles
      const int pt = jj % kPTiles;
      if (jj >= kPTiles) {
        if (!wwait(&bar->o_done[pt], ((jj / kPTiles) - 1) & 1)) { ok = false; break; }
        if (!wwait(&bar->p_free[pt], ((jj / kPTiles) - 1) & 1)) { ok = false; break; }
      }
      {
        const uint32_t prow = pt * kPBytes + r * 128;
        unsigned char* own = p_s + prow;
#pragma unroll
        for (int k4 = 0; k4 < 4; ++k4) {
          const uint32_t off = ((4 * c + k4) ^ (r & 7)) << 4;   // 128-byte swizzle of the UMMA K-major tile
          const uint4 v = make_uint4(pk[4 * k4], pk[4 * k4 + 1], pk[4 * k4 + 2], pk[4 * k4 + 3]);
          *reinterpret_cast<uint4*>(own + off) = v;
          st_async_v4(p_peer + prow + off, v, pfull_peer + pt * 8);
        }
      }
      // cache slots past the sequence (or a page never loaded) feed the value
      // product: zero their latent columns so that 0 * garbage cannot make NaN
      if (nvalid < 64) {
        unsigned char* pgb = pg_s + st * kPageBytes;
        const int nz = (64 - nvalid) * 4 * 8;           // 16-byte chunks to clear
        for (int t = ltid; t < nz; t += 128) {
          const int row = nvalid + t / 32, blk = (t / 8) & 3, ch = t & 7;
          *reinterpret_cast<uint4*>(pgb + blk * 8192 + row * 128 + ch * 16) = make_uint4(0, 0, 0, 0);
        }
      }
      fence_proxy_async_smem();                        // own P / zeroed rows -> tensor core
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (warp == 6) mbar_arrive_expect_tx(&bar->p_full[pt], kPBytes / 2);  // the peer's half
        else mbar_arrive(&bar->p_full[pt]);
      }

      if (cb.last()) {
        // epilogue: O / l and lse of this piece, l summed over the two key halves
        if (leader) mbar_arrive_expect_tx(&bar->l_full, 128 * 4);
        st_async_b32(lrecv_peer + r * 4, __float_as_uint(l), lfull_peer);
        if (!wwait(&bar->l_full, cb.p & 1)) { ok = false; break; }
        const float lt = l + l_recv[r];
        if (!wwait(&bar->o_done[pt], (jj / kPTiles) & 1)) { ok = false; break; }
        tc_fence_after();
        const float inv_l = lt > 0.f ? 1.f / lt : 0.f;
        const int grow_row = row0 + r;
        float* dst = a.part_o + ((size_t)cb.pc.id * prm.rows_total + grow_row) * a.d_c + c * 256;
#pragma unroll 1
        for (int cc = 0; cc < 256; cc += 32) {
          float o[32];
          tmem_ld32(tmem + lane_off + cc, o);
          tmem_wait_ld();
          if (row_valid) {
#pragma unroll
            for (int i = 0; i < 32; i += 4)
              *reinterpret_cast<float4*>(dst + cc + i) =
                  make_float4(o[i] * inv_l, o[i + 1] * inv_l, o[i + 2] * inv_l, o[i + 3] * inv_l);
          }
        }
        if (row_valid && c == 0)
          a.part_lse[(size_t)cb.pc.id * prm.rows_total + grow_row] =
              lt > 0.f ? (m_used + log2f(lt)) * 0.6931471805599453f : -INFINITY;
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar->o_free);
      }
    }
  }

  // ------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  __syncwarp();
  cluster_sync();  // the peer no longer stores into this CTA's shared memory
  if (*abort_flag) {
    // after a time-out the peer may have stores to this CTA still in flight
    // (its waits for them gave up): give them time to land before exiting
    const long long t0 = clock64();
    while (clock64() - t0 < 200000) __nanosleep(1000);
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------------ host side

}  // namespace

bool decode_tc_supported(int d_c, int d_rope, int page_size) { return d_c == 512 && d_rope == 64 && page_size == 64; }

int decode_tc_workers(int sms, int rows_total) {
  const int tiles = (rows_total + 127) / 128;
  const int g = (sms / 2) / tiles;
  return g < 1 ? 1 : g;
}

cudaError_t launch_decode_split_tc(const DecodeArgs& a, long long spin_limit, cudaStream_t stream) {
  const int rows_total = a.nq * a.n_heads;
  CUtensorMap tq64, tp128, tp64;
  const uint64_t qrows = (uint64_t)a.batch * rows_total;
  const uint64_t prows = (uint64_t)a.num_pages * 64;
  if (!encode_rows576(&tq64, a.q_lat, qrows, 32, 128, CU_TENSOR_MAP_SWIZZLE_64B) ||
      !encode_rows576(&tp128, a.pool, prows, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_rows576(&tp64, a.pool, prows, 32, 64, CU_TENSOR_MAP_SWIZZLE_64B))
    return cudaErrorInvalidValue;
  TcParams prm;
  prm.d = a;
  prm.rows_total = rows_total;
  prm.scale_log2 = a.scale * 1.4426950408889634f;
  prm.spin_limit = spin_limit;
  cudaError_t e = cudaFuncSetAttribute(decode_split_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kSmemBytes);
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
  e = cudaLaunchKernelEx(&cfg, decode_split_tc_kernel, tq64, tp128, tp64, prm);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace mla
