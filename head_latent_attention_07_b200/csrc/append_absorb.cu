// mla_append_latent and mla_absorb_q kernels.
//
// append:  [c_t || k^_t] = w_dkv h_t (c_t = W_DKV h_t, k^_t = W_KR h_t), k_t^R =
//          RoPE(k^_t, pos_t); the bf16 row goes to its paged cache slot.
// absorb:  q_lat[t][h] = [W_UK,h^T q_nope || RoPE(q_rope, pos_t)].
// Both are weight-read bound (w_dkv 8.3 MB, W_UK 16.8 MB at DeepSeek-V3 shape):
// each CTA streams its slice of the weights once and applies it to a block of
// up to 16 tokens held on chip.
#include "common.cuh"
#include "decode.h"
#include "mma_frag.cuh"

namespace mla {

namespace {

constexpr int kTokBlk = 16;

// ------------------------------------------------------------------ append
// [c || k^] rows = w_dkv [R x D] . h^T [D x T] on the tensor cores: one CTA per
// 16-row tile of w_dkv and 16 tokens; its 8 warps split the reduction over D
// in 32-wide slices (mma_frag.cuh), their partial tiles are summed in shared
// memory, then RoPE is applied to the k^ rows and the bf16 row goes to its slot.
constexpr int kAppWarps = 8;
constexpr int kAppSplit = 8;   // CTAs of a cluster splitting the reduction over D

__global__ void __launch_bounds__(kAppWarps * 32)
append_latent_kernel(AppendArgs a) {
  __shared__ float part[kAppWarps][16][17];
  __shared__ float red[kAppSplit][16][17];   // cluster leader: the split CTAs' tiles
  // split cluster barrier: the wait before the first remote store below makes sure
  // every CTA of the cluster (the leader included) has started
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
  const int R = a.d_c + a.d_rope;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, q = lane & 3;
  const int m0 = blockIdx.x * 16;
  const int t0 = blockIdx.y * kTokBlk;
  uint32_t split;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(split));
  const int ra_row = m0 + g, rb_row = m0 + g + 8;
  const int ta = t0 + g, tb = t0 + g + 8;
  const uint4 z = make_uint4(0, 0, 0, 0);
  float d0[4] = {0.f, 0.f, 0.f, 0.f}, d1[4] = {0.f, 0.f, 0.f, 0.f};
  const int nslices = (a.d_model + 31) / 32;
  // slices of this CTA's eighth, interleaved over its warps; 4 per batch of loads
  constexpr int kStride = 4 * kAppWarps * kAppSplit;
  uint4 ra[4], rb[4];
  auto load_w = [&](int base) {
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int sl = base + u * kAppWarps * kAppSplit;
      const int kk = sl * 32 + 8 * q;
      const bool kin = sl < nslices && kk < a.d_model;
      ra[u] = (kin && ra_row < R) ? ldg_stream(a.w_dkv + (size_t)ra_row * a.d_model + kk) : z;
      rb[u] = (kin && rb_row < R) ? ldg_stream(a.w_dkv + (size_t)rb_row * a.d_model + kk) : z;
    }
  };
  // The weights are read before the dependency wait, while the preceding kernel
  // on the stream finishes (no kernel of this library writes weights; the header
  // states the caller's side: the kernel enqueued just before the call must not
  // write them).
  load_w(split * kAppWarps + warp);
  grid_dependency_wait();   // h, the page table and the pool may be written by the preceding kernel
  allow_dependent_launch();
  for (int base = split * kAppWarps + warp; base < nslices; base += kStride) {
    uint4 ha[4], hb[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int sl = base + u * kAppWarps * kAppSplit;
      const int kk = sl * 32 + 8 * q;
      const bool kin = sl < nslices && kk < a.d_model;
      ha[u] = (kin && ta < a.n_tokens) ? *reinterpret_cast<const uint4*>(a.h + (size_t)ta * a.d_model + kk) : z;
      hb[u] = (kin && tb < a.n_tokens) ? *reinterpret_cast<const uint4*>(a.h + (size_t)tb * a.d_model + kk) : z;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      mma_k32(d0, ra[u], rb[u], ha[u]);
      mma_k32(d1, ra[u], rb[u], hb[u]);
    }
    if (base + kStride < nslices) load_w(base + kStride);
  }
  // fragment -> part[warp][row][token]
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int row = g + ((e & 2) ? 8 : 0), tok = 2 * q + (e & 1);
    part[warp][row][tok] = d0[e];
    part[warp][row][tok + 8] = d1[e];
  }
  __syncthreads();
  asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
  {
    // this CTA's tile -> slot `split` of the leader's shared memory
    const int row = threadIdx.x >> 4, tok = threadIdx.x & 15;
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < kAppWarps; ++w) v += part[w][row][tok];
    const uint32_t local = static_cast<uint32_t>(__cvta_generic_to_shared(&red[split][row][tok]));
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, 0;" : "=r"(remote) : "r"(local));
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(remote), "f"(v) : "memory");
  }
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
  if (split != 0) return;
  __shared__ float vals[16][17];
  {
    const int row = threadIdx.x >> 4, tok = threadIdx.x & 15;
    float v = 0.f;
#pragma unroll
    for (int sp = 0; sp < kAppSplit; ++sp) v += red[sp][row][tok];
    vals[row][tok] = v;
  }
  __syncthreads();
  // store: thread (row, token); RoPE rows pair up inside the tile (m0 and d_c are even)
  const int rr = threadIdx.x >> 4, j = threadIdx.x & 15;
  const int row = m0 + rr, t = t0 + j;
  if (row >= R || t >= a.n_tokens) return;
  const int seq = a.seq_idx[t], p = a.pos[t];
  if (seq < 0 || seq >= a.batch || p < 0 || p >= a.max_pages * a.page_size) {
    record_status(a.dev_status, MLA_ERR_RANGE);
    return;
  }
  const int page = a.page_table[(size_t)seq * a.max_pages + p / a.page_size];
  if (page < 0 || page >= a.num_pages) {
    record_status(a.dev_status, MLA_ERR_RANGE);
    return;
  }
  float val = vals[rr][j];
  if (row >= a.d_c) {
    const int qch = row - a.d_c;          // channel within the RoPE key
    float c, s;
    rope_cos_sin(p, a.inv_freq[qch >> 1], &c, &s);
    const float x0 = vals[rr & ~1][j], x1 = vals[rr | 1][j];
    val = (qch & 1) ? x0 * s + x1 * c : x0 * c - x1 * s;
  }
  a.pool[((size_t)page * a.page_size + p % a.page_size) * R + row] = f32_to_bf16(val);
}

// ------------------------------------------------------------------ absorb
constexpr int kAbsThreads = 256;
constexpr int kAbsMaxKSteps = 12;   // tensor-core path: qk_nope <= 192

// RoPE(q_rope, pos) of one head for up to kTokBlk tokens, by threads tid of nthreads.
__device__ __forceinline__ void absorb_rope_part(const AbsorbArgs& a, int h, int t0, int tid, int nthreads) {
  const int dq = a.qk_nope + a.d_rope;
  const int R = a.d_c + a.d_rope;
  const int npair = a.d_rope / 2;
  for (int idx = tid; idx < kTokBlk * npair; idx += nthreads) {
    const int k = idx / npair, i = idx % npair;
    const int t = t0 + k;
    if (t >= a.n_tokens) continue;
    const uint16_t* src = a.q + ((size_t)t * a.n_heads + h) * dq + a.qk_nope + 2 * i;
    const float x0 = bf16_to_f32(src[0]), x1 = bf16_to_f32(src[1]);
    float c, s;
    rope_cos_sin(a.pos[t], a.inv_freq[i], &c, &s);
    *reinterpret_cast<uint32_t*>(a.q_lat + ((size_t)t * a.n_heads + h) * R + a.d_c + 2 * i) =
        pack_bf16x2(x0 * c - x1 * s, x0 * s + x1 * c);
  }
}

// q~ = W_UK,h^T q_nope on the tensor cores, one CTA per (head, run of
// blocks_per_cta 16-token blocks): per block D^T [16 tokens x d_c] = Q [16 x
// qk_nope] . W_UK,h [qk_nope x d_c].  W_UK,h is staged in shared memory once
// (rows padded by 16 bytes) and read as B fragments with ldmatrix.trans; each of
// the 8 warps owns d_c / 8 output columns.
__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t* r) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__global__ void __launch_bounds__(kAbsThreads)
absorb_q_mma_kernel(AbsorbArgs a) {
  extern __shared__ __align__(16) uint16_t wsm[];   // [qk_nope][d_c + 8]
  const int h = blockIdx.x;
  const int dq = a.qk_nope + a.d_rope;
  const int R = a.d_c + a.d_rope;
  const int ws = a.d_c + 8;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, q4 = lane & 3;
  // stage W_UK,h
  const uint16_t* wh = a.w_uk + (size_t)h * a.qk_nope * a.d_c;
  const int cpr = a.d_c / 8;                        // 16-byte chunks per row
  for (int idx = threadIdx.x; idx < a.qk_nope * cpr; idx += blockDim.x) {  // all copies in flight at once
    const int i = idx / cpr, cch = idx % cpr;
    const uint32_t dst = static_cast<uint32_t>(__cvta_generic_to_shared(wsm + i * ws + cch * 8));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(wh + (size_t)i * a.d_c + cch * 8)
                 : "memory");
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
  // W_UK,h streams in before the dependency wait, while the preceding kernel on
  // the stream finishes (as in the append kernel above).
  grid_dependency_wait();   // q may be written by the preceding kernel
  allow_dependent_launch();
  const int nblk = (a.n_tokens + kTokBlk - 1) / kTokBlk;
  const int blk_end = min(nblk, ((int)blockIdx.y + 1) * a.blocks_per_cta);
  for (int blk = blockIdx.y * a.blocks_per_cta; blk < blk_end; ++blk) {
  const int t0 = blk * kTokBlk;
  // A fragments (q_nope of this warp's 16 tokens) for every k step, loaded once
  // per block (the first while W_UK,h streams in)
  const int ta = t0 + g, tb = t0 + g + 8;
  const uint16_t* qa = a.q + ((size_t)ta * a.n_heads + h) * dq;
  const uint16_t* qb = a.q + ((size_t)tb * a.n_heads + h) * dq;
  const bool va = ta < a.n_tokens, vb = tb < a.n_tokens;
  const int nks = a.qk_nope / 16;
  uint32_t af[kAbsMaxKSteps][4];
#pragma unroll
  for (int k = 0; k < kAbsMaxKSteps; ++k) {
    const int ia = 16 * k + 2 * q4;
    const bool kin = k < nks;
    af[k][0] = (kin && va) ? *reinterpret_cast<const uint32_t*>(qa + ia) : 0u;
    af[k][1] = (kin && vb) ? *reinterpret_cast<const uint32_t*>(qb + ia) : 0u;
    af[k][2] = (kin && va) ? *reinterpret_cast<const uint32_t*>(qa + ia + 8) : 0u;
    af[k][3] = (kin && vb) ? *reinterpret_cast<const uint32_t*>(qb + ia + 8) : 0u;
  }
  absorb_rope_part(a, h, t0, threadIdx.x, blockDim.x);
  if (blk == blockIdx.y * a.blocks_per_cta) {
    asm volatile("cp.async.wait_all;" ::: "memory");
    __syncthreads();
  }
  const int ntiles = a.d_c / 8;
  for (int nt0 = warp * 2; nt0 < ntiles; nt0 += 16) {  // pairs of 8-column tiles
    float d[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    const int j0 = nt0 * 8;
#pragma unroll
    for (int k = 0; k < kAbsMaxKSteps; ++k) {
      if (k >= nks) break;
      const int i0 = 16 * k;
      const uint32_t a0 = af[k][0], a1 = af[k][1], a2 = af[k][2], a3 = af[k][3];
      // tiles: 0 = W[i0..+8][j0..+8], 1 = W[i0+8..][j0..], 2 = W[i0..][j0+8..], 3 = W[i0+8..][j0+8..]
      const int tile = lane >> 3, rr = lane & 7;
      const int wi = i0 + rr + ((tile & 1) ? 8 : 0);
      const int wj = j0 + ((tile & 2) ? 8 : 0);
      uint32_t b[4];
      ldsm_x4_trans(static_cast<uint32_t>(__cvta_generic_to_shared(wsm + wi * ws + wj)), b);
      mma_16816(d[0], a0, a1, a2, a3, b[0], b[1]);
      if (nt0 + 1 < ntiles) mma_16816(d[1], a0, a1, a2, a3, b[2], b[3]);
    }
#pragma unroll
    for (int n = 0; n < 2; ++n) {
      const int j = j0 + 8 * n + 2 * q4;
      if (nt0 + n >= ntiles) continue;
      if (va) *reinterpret_cast<uint32_t*>(a.q_lat + ((size_t)ta * a.n_heads + h) * R + j) = pack_bf16x2(d[n][0], d[n][1]);
      if (vb) *reinterpret_cast<uint32_t*>(a.q_lat + ((size_t)tb * a.n_heads + h) * R + j) = pack_bf16x2(d[n][2], d[n][3]);
    }
  }
  }   // token blocks
}

// CUDA-core fallback for shapes whose W_UK,h does not fit in shared memory.
__global__ void __launch_bounds__(kAbsThreads)
absorb_q_kernel(AbsorbArgs a) {
  extern __shared__ __align__(16) float qn[];   // [kTokBlk][qk_nope]
  grid_dependency_wait();
  allow_dependent_launch();
  const int h = blockIdx.x;
  const int t0 = blockIdx.y * kTokBlk;
  const int dq = a.qk_nope + a.d_rope;
  const int R = a.d_c + a.d_rope;
  for (int idx = threadIdx.x; idx < kTokBlk * a.qk_nope; idx += blockDim.x) {
    const int j = idx / a.qk_nope, i = idx % a.qk_nope;
    const int t = t0 + j;
    qn[idx] = t < a.n_tokens ? bf16_to_f32(a.q[((size_t)t * a.n_heads + h) * dq + i]) : 0.f;
  }
  __syncthreads();
  const uint16_t* wh = a.w_uk + (size_t)h * a.qk_nope * a.d_c;
  // content part: thread owns column pairs (j, j+1)
  for (int j = 2 * threadIdx.x; j < a.d_c; j += 2 * blockDim.x) {
    float acc0[kTokBlk], acc1[kTokBlk];
#pragma unroll
    for (int k = 0; k < kTokBlk; ++k) { acc0[k] = 0.f; acc1[k] = 0.f; }
    for (int i = 0; i < a.qk_nope; ++i) {
      const uint32_t w2 = *reinterpret_cast<const uint32_t*>(wh + (size_t)i * a.d_c + j);
      const float w0 = bf16_lo(w2), w1 = bf16_hi(w2);
#pragma unroll
      for (int k = 0; k < kTokBlk; ++k) {
        const float qv = qn[k * a.qk_nope + i];
        acc0[k] += w0 * qv;
        acc1[k] += w1 * qv;
      }
    }
#pragma unroll
    for (int k = 0; k < kTokBlk; ++k) {
      const int t = t0 + k;
      if (t < a.n_tokens)
        *reinterpret_cast<uint32_t*>(a.q_lat + ((size_t)t * a.n_heads + h) * R + j) =
            pack_bf16x2(acc0[k], acc1[k]);
    }
  }
  absorb_rope_part(a, h, t0, threadIdx.x, blockDim.x);
}

// ------------------------------------------------------------------ append + absorb in one launch
// A decode step's two prologue calls on the same <= 16 tokens are independent:
// one launch runs both, so that neither waits for the other.  CTA i < H absorbs
// head i's queries with warps 0-7 (as absorb_q_mma_kernel, one 16-token block);
// every CTA also computes with warps 8-15 up to kFusedMaxRows rows of [c || k^]
// (whole RoPE pairs: the R / 2 pairs are dealt evenly to the CTAs) for all the
// tokens: 32-wide slices of d_model dealt to the warps (rows g < 8 of the
// mma.sync tile), the warps' tiles summed in shared memory, then RoPE and the
// store as in append_latent_kernel.  Weights (W_UK,h and the rows of w_dkv) are
// read before the dependency wait.
constexpr int kFusedThreads = 512;
constexpr int kFusedMaxRows = 8;

__device__ __forceinline__ void role_sync(int id) {
  asm volatile("bar.sync %0, 256;" ::"r"(id) : "memory");   // the 8 warps of one role
}

__global__ void __launch_bounds__(kFusedThreads, 1)
append_absorb_kernel(AppendArgs ap, AbsorbArgs ab, int npairs) {
  extern __shared__ __align__(16) uint16_t wsm[];          // absorb: [qk_nope][d_c + 8]
  __shared__ float part[8][kFusedMaxRows][17];             // append: per warp [row][token]
  __shared__ float vals[kFusedMaxRows][17];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, q4 = lane & 3;
  const int h = blockIdx.x;
  const bool absorb_cta = h < ab.n_heads;
  const int R = ap.d_c + ap.d_rope;
  const int D = ap.d_model;
  const int T = ap.n_tokens;
  const int nslices = (D + 31) / 32;
  const int p0 = (int)(((long long)npairs * blockIdx.x) / gridDim.x);
  const int p1 = (int)(((long long)npairs * (blockIdx.x + 1)) / gridDim.x);
  const int r0 = 2 * p0, nrows = 2 * (p1 - p0);          // <= kFusedMaxRows
  const int ws = ab.d_c + 8;
  const uint4 z = make_uint4(0, 0, 0, 0);

  // ---- before the dependency wait: weights only
  if (warp < 8 && absorb_cta) {
    const uint16_t* wh = ab.w_uk + (size_t)h * ab.qk_nope * ab.d_c;
    const int cpr = ab.d_c / 8;
    for (int idx = threadIdx.x; idx < ab.qk_nope * cpr; idx += 256) {
      const int i = idx / cpr, cch = idx % cpr;
      const uint32_t dst = static_cast<uint32_t>(__cvta_generic_to_shared(wsm + i * ws + cch * 8));
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(wh + (size_t)i * ab.d_c + cch * 8)
                   : "memory");
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  }
  const int aw = warp - 8;                                   // append warp 0..7
  uint4 ra[4];
  auto load_w = [&](int base) {
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int sl = base + 8 * u;
      const int kk = 32 * sl + 8 * q4;
      ra[u] = (sl < nslices && kk < D && g < nrows) ? ldg_stream(ap.w_dkv + (size_t)(r0 + g) * D + kk) : z;
    }
  };
  if (warp >= 8) load_w(aw);
  grid_dependency_wait();   // h, q, the page table and the pool may be written by the preceding kernel
  allow_dependent_launch();

  if (warp >= 8) {
    // ---- append: rows [r0, r0 + nrows) for all T tokens
    float d0[4] = {0.f, 0.f, 0.f, 0.f}, d1[4] = {0.f, 0.f, 0.f, 0.f};
    for (int base = aw; base < nslices; base += 32) {
      uint4 ha[4], hb[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int sl = base + 8 * u;
        const int kk = 32 * sl + 8 * q4;
        const bool kin = sl < nslices && kk < D;
        ha[u] = (kin && g < T) ? *reinterpret_cast<const uint4*>(ap.h + (size_t)g * D + kk) : z;
        hb[u] = (kin && g + 8 < T) ? *reinterpret_cast<const uint4*>(ap.h + (size_t)(g + 8) * D + kk) : z;
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        mma_k32(d0, ra[u], z, ha[u]);
        mma_k32(d1, ra[u], z, hb[u]);
      }
      if (base + 32 < nslices) load_w(base + 32);
    }
    // fragment: row g, tokens 2 q4 + {0, 1} of each 8-token tile (rows g + 8 are empty)
    part[aw][g][2 * q4] = d0[0];
    part[aw][g][2 * q4 + 1] = d0[1];
    part[aw][g][8 + 2 * q4] = d1[0];
    part[aw][g][8 + 2 * q4 + 1] = d1[1];
    role_sync(1);
    const int at = threadIdx.x - 256;
    const int rr = at >> 4, j = at & 15;                    // 8 rows x 16 tokens over the first 128 threads
    if (at < kFusedMaxRows * 16) {
      float v = 0.f;
#pragma unroll
      for (int w = 0; w < 8; ++w) v += part[w][rr][j];
      vals[rr][j] = v;
    }
    role_sync(1);
    if (at < kFusedMaxRows * 16 && rr < nrows && j < T) {
      const int row = r0 + rr, t = j;
      const int seq = ap.seq_idx[t], p = ap.pos[t];
      bool ok = seq >= 0 && seq < ap.batch && p >= 0 && p < ap.max_pages * ap.page_size;
      const int page = ok ? ap.page_table[(size_t)seq * ap.max_pages + p / ap.page_size] : -1;
      ok = ok && page >= 0 && page < ap.num_pages;
      if (!ok) {
        record_status(ap.dev_status, MLA_ERR_RANGE);
      } else {
        float val = vals[rr][j];
        if (row >= ap.d_c) {
          const int qch = row - ap.d_c;                    // channel within the RoPE key
          float c, sn;
          rope_cos_sin(p, ap.inv_freq[qch >> 1], &c, &sn);
          const float x0 = vals[rr & ~1][j], x1 = vals[rr | 1][j];
          val = (qch & 1) ? x0 * sn + x1 * c : x0 * c - x1 * sn;
        }
        ap.pool[((size_t)page * ap.page_size + p % ap.page_size) * R + row] = f32_to_bf16(val);
      }
    }
  } else if (absorb_cta) {
    // ---- absorb: head h, tokens [0, T)
    const int dq = ab.qk_nope + ab.d_rope;
    const uint16_t* qa = ab.q + ((size_t)g * ab.n_heads + h) * dq;
    const uint16_t* qb = ab.q + ((size_t)(g + 8) * ab.n_heads + h) * dq;
    const bool va = g < ab.n_tokens, vb = g + 8 < ab.n_tokens;
    const int nks = ab.qk_nope / 16;
    uint32_t af[kAbsMaxKSteps][4];
#pragma unroll
    for (int k = 0; k < kAbsMaxKSteps; ++k) {
      const int ia = 16 * k + 2 * q4;
      const bool kin = k < nks;
      af[k][0] = (kin && va) ? *reinterpret_cast<const uint32_t*>(qa + ia) : 0u;
      af[k][1] = (kin && vb) ? *reinterpret_cast<const uint32_t*>(qb + ia) : 0u;
      af[k][2] = (kin && va) ? *reinterpret_cast<const uint32_t*>(qa + ia + 8) : 0u;
      af[k][3] = (kin && vb) ? *reinterpret_cast<const uint32_t*>(qb + ia + 8) : 0u;
    }
    absorb_rope_part(ab, h, 0, threadIdx.x, 256);
    asm volatile("cp.async.wait_all;" ::: "memory");
    role_sync(2);
    const int Rq = ab.d_c + ab.d_rope;
    const int ntiles = ab.d_c / 8;
    for (int nt0 = warp * 2; nt0 < ntiles; nt0 += 16) {      // pairs of 8-column tiles
      float d[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
      const int j0 = nt0 * 8;
#pragma unroll
      for (int k = 0; k < kAbsMaxKSteps; ++k) {
        if (k >= nks) break;
        const int i0 = 16 * k;
        const int tile = lane >> 3, rr = lane & 7;
        const int wi = i0 + rr + ((tile & 1) ? 8 : 0);
        const int wj = j0 + ((tile & 2) ? 8 : 0);
        uint32_t b[4];
        ldsm_x4_trans(static_cast<uint32_t>(__cvta_generic_to_shared(wsm + wi * ws + wj)), b);
        mma_16816(d[0], af[k][0], af[k][1], af[k][2], af[k][3], b[0], b[1]);
        if (nt0 + 1 < ntiles) mma_16816(d[1], af[k][0], af[k][1], af[k][2], af[k][3], b[2], b[3]);
      }
#pragma unroll
      for (int n = 0; n < 2; ++n) {
        const int j = j0 + 8 * n + 2 * q4;
        if (nt0 + n >= ntiles) continue;
        if (va) *reinterpret_cast<uint32_t*>(ab.q_lat + ((size_t)g * ab.n_heads + h) * Rq + j) = pack_bf16x2(d[n][0], d[n][1]);
        if (vb) *reinterpret_cast<uint32_t*>(ab.q_lat + ((size_t)(g + 8) * ab.n_heads + h) * Rq + j) = pack_bf16x2(d[n][2], d[n][3]);
      }
    }
  }
}

}  // namespace

cudaError_t launch_append_latent(const AppendArgs& a, cudaStream_t stream) {
  const int R = a.d_c + a.d_rope;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((R + 15) / 16, (a.n_tokens + kTokBlk - 1) / kTokBlk, kAppSplit);
  cfg.blockDim = dim3(kAppWarps * 32, 1, 1);
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = kAppSplit;
  attr[1] = pdl_attribute();
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  cudaError_t e = cudaLaunchKernelEx(&cfg, append_latent_kernel, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_absorb_q(const AbsorbArgs& a, cudaStream_t stream) {
  const int nblk = (a.n_tokens + kTokBlk - 1) / kTokBlk;
  const int per = a.blocks_per_cta < 1 ? 1 : a.blocks_per_cta;
  dim3 grid(a.n_heads, (nblk + per - 1) / per);
  const size_t wsmem = (size_t)a.qk_nope * (a.d_c + 8) * 2;
  cudaLaunchAttribute attr[1] = {pdl_attribute()};
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kAbsThreads, 1, 1);
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (a.qk_nope % 16 == 0 && a.qk_nope <= 16 * kAbsMaxKSteps && a.d_c % 8 == 0 && wsmem <= 200 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(absorb_q_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)wsmem);
    if (e != cudaSuccess) return e;
    cfg.dynamicSmemBytes = wsmem;
    e = cudaLaunchKernelEx(&cfg, absorb_q_mma_kernel, a);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
  }
  const size_t smem = (size_t)kTokBlk * a.qk_nope * 4;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(absorb_q_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  cfg.gridDim = dim3(a.n_heads, nblk, 1);   // one 16-token block per CTA
  cfg.dynamicSmemBytes = smem;
  cudaError_t e = cudaLaunchKernelEx(&cfg, absorb_q_kernel, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

bool append_absorb_fusable(const AppendArgs& ap, const AbsorbArgs& ab) {
  const size_t wsmem = (size_t)ab.qk_nope * (ab.d_c + 8) * 2;
  return ap.n_tokens <= kTokBlk && ab.n_tokens == ap.n_tokens && ab.qk_nope % 16 == 0 &&
         ab.qk_nope <= 16 * kAbsMaxKSteps && ab.d_c % 8 == 0 && wsmem <= 180 * 1024 &&
         (ap.d_c + ap.d_rope) % 2 == 0;
}

cudaError_t launch_append_absorb(const AppendArgs& ap, const AbsorbArgs& ab, cudaStream_t stream) {
  if (!append_absorb_fusable(ap, ab)) {
    cudaError_t e = launch_append_latent(ap, stream);
    if (e != cudaSuccess) return e;
    return launch_absorb_q(ab, stream);
  }
  const int npairs = (ap.d_c + ap.d_rope) / 2;
  const int need = (npairs + kFusedMaxRows / 2 - 1) / (kFusedMaxRows / 2);   // CTAs with <= 8 rows each
  const int ctas = ab.n_heads > need ? ab.n_heads : need;
  const size_t wsmem = (size_t)ab.qk_nope * (ab.d_c + 8) * 2;
  cudaError_t e = cudaFuncSetAttribute(append_absorb_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)wsmem);
  if (e != cudaSuccess) return e;
  cudaLaunchAttribute attr[1] = {pdl_attribute()};
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(ctas, 1, 1);
  cfg.blockDim = dim3(kFusedThreads, 1, 1);
  cfg.dynamicSmemBytes = wsmem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, append_absorb_kernel, ap, ab, npairs);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace mla
