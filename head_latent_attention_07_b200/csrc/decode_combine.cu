// Combine of the split-KV partials, then the W_UV up-projection.
//
// For query row (token t, head h) with pieces s of its sequence:
//   LSE   = ln sum_s exp(lse_s)
//   o_lat = sum_s exp(lse_s - LSE) * O_s          (O_s already normalised per piece)
//   out[t][h][v] = sum_c W_UV[h][v][c] * o_lat[c]  (values up-projected once, after
//                                                   attending over latents)
// Work split: one CTA per (head, group of 16 query tokens) over all d_c latent
// columns.  Its 512 threads merge the partials (32 per token, each owning 16
// columns; each partial byte is read once, by one CTA) and write the merged
// rows, split into two bf16 terms (hi + lo, which keep about 16 bits of the
// fp32 mantissa), as the 32 rows of the B operand of one tcgen05 MMA chain:
// D[128 out rows x 32] = W_UV,h chunk [128 x d_c] . [hi rows; lo rows]^T, fp32
// in TMEM, d_c / 16 MMAs issued by one thread.  Four warps read D back (one TMEM
// lane quarter each: 32 out rows) and store hi + lo.  W_UV,h (a chunk of 128 out
// rows) is staged in shared memory by cp.async, in the 128-byte swizzled
// K-major layout the MMA reads, before the kernel waits for the split kernel's
// partials, so after that wait only the merge, the MMAs and the stores remain.
//
// Context split (one call per rank over a window of every sequence's pages):
// with a.out_lat set, the kernel stops after the merge and writes the rank's
// o_lat and lse; the rank-merge form (RANKS) then takes the ranks' partials as
// its pieces (plain loads through the given pointers, which may point into a
// peer GPU's memory) and finishes with W_UV as above.
#include "common.cuh"
#include "decode.h"
#include "mma_frag.cuh"
#include "plan.cuh"
#include "sm100.cuh"

namespace mla {

namespace {

using namespace sm100;

constexpr int kThreads = 512;
constexpr int kTok = 16;       // query tokens per CTA
constexpr int kCols = 512;     // latent columns per CTA (d_c <= 512)
constexpr int kVChunk = 128;   // out rows per round (8 row tiles x 16)
constexpr int kPieceBatch = 4;         // pieces whose loads are in flight at once
// MMA operands in shared memory, K-major, 128-byte swizzle: blocks of 64 latent
// columns, 128 bytes per row, 16-byte chunk c of row r at chunk c ^ (r mod 8)
constexpr int kKBlocks = kCols / 64;
constexpr int kWBlock = kVChunk * 128;        // [128 out rows x 64 columns] of W_UV
constexpr int kOBlock = 2 * kTok * 128;       // [32 rows (hi, lo) x 64 columns] of the merged rows
constexpr uint32_t kTmemCols = 32;

// One lane of the (converged) warp returns true.
__device__ __forceinline__ bool elect_lane() {
  uint32_t is_leader;
  asm volatile("{\n\t.reg .pred p;\n\telect.sync _|p, 0xffffffff;\n\tselp.u32 %0, 1, 0, p;\n\t}" : "=r"(is_leader));
  return is_leader != 0;
}

__device__ __forceinline__ uint32_t swz(int row, int chunk) {
  return uint32_t(row * 128 + ((chunk ^ (row & 7)) << 4));
}

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

template <bool RANKS>
__global__ void __launch_bounds__(kThreads, 1)
decode_combine_kernel(DecodeArgs a, const __grid_constant__ RankSources src) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  // swizzled operand blocks first, on a 1024-byte boundary
  unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t w_s = smem_addr(sm);                      // kKBlocks x kWBlock
  const uint32_t o_s = w_s + kKBlocks * kWBlock;           // kKBlocks x kOBlock
  PlanSmem* ps = reinterpret_cast<PlanSmem*>(sm + kKBlocks * (kWBlock + kOBlock));
  uint64_t* mma_bar = reinterpret_cast<uint64_t*>(reinterpret_cast<unsigned char*>(ps) +
                                                  ((sizeof(PlanSmem) + 15) & ~size_t(15)));
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(mma_bar + 1);

  const int h = blockIdx.x;
  const int t0 = blockIdx.y * kTok;
  const int T = a.batch * a.nq;
  const int rows_total = a.nq * a.n_heads;
  const int ncol = a.d_c;                       // multiple of 8, <= kCols
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, q = lane & 3;
  const uint16_t* wh = a.w_uv + (size_t)h * a.v_head * a.d_c;
  // W_UV,h rows [v0, v0 + kVChunk) -> the swizzled A operand (zeros outside the matrix)
  auto stage_w = [&](int v0) {
    for (int idx = tid; idx < kVChunk * (kCols / 8); idx += kThreads) {
      const int vl = idx / (kCols / 8), cc8 = idx % (kCols / 8), cc = 8 * cc8;
      const uint32_t dst = w_s + (cc8 >> 3) * kWBlock + swz(vl, cc8 & 7);
      if (v0 + vl < a.v_head && cc < ncol) {
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst),
                     "l"(wh + (size_t)(v0 + vl) * a.d_c + cc)
                     : "memory");
      } else {
        asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(dst), "r"(0u) : "memory");
      }
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  const bool lat_mode = !RANKS && a.out_lat != nullptr;
  if (!lat_mode) {   // the latent form stops after the merge: no MMA, no TMEM
    if (tid == 0) {
      mbar_init(mma_bar, 1);
      fence_mbar_init();
    }
    if (warp == 0) {
      tmem_alloc(tmem_holder, kTmemCols);
      tmem_relinquish();
    }
  }

  if (RANKS) {
    // the predecessor is the caller's: only the weight rows are read before the
    // wait (the kernel enqueued just before the call must not write W_UV)
    stage_w(0);
    grid_dependency_wait();
  } else {
    // The predecessor on the stream is always this call's split kernel, which
    // writes only the partials and lets this kernel launch only after its own
    // dependency wait: seq_lens and W_UV are final here, the partials after the
    // wait below.
    if (!lat_mode) stage_w(0);
    build_plan(ps, a.seq_lens, a.batch, a.nq, a.max_pages, a.page_size, a.G, a.piece_cost, nullptr, a.kv_rank,
               a.kv_ranks);
    grid_dependency_wait();   // the split kernel's partials
  }
  allow_dependent_launch();   // after the wait, as in every kernel here

  // 1. merge: 32 threads per token, each owning columns [8 gc, 8 gc + 8) and
  //    [256 + 8 gc, 256 + 8 gc + 8); one pass over the pieces in batches (their
  //    LSEs and partial rows loaded together), with the running max moved as
  //    batches arrive
  {
    const int j = tid >> 5, gc = tid & 31;
    const int t = t0 + j;
    float acc[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) acc[e] = 0.f;
    bool cols[2];
#pragma unroll
    for (int half = 0; half < 2; ++half) cols[half] = 256 * half + 8 * gc < ncol;
    if (t < T) {
      const int b = t / a.nq, i = t % a.nq;
      const int row = i * a.n_heads + h;
      const size_t trow = (size_t)t * a.n_heads + h;   // row of a rank's partial [T, H, d_c]
      const int pb = RANKS ? 0 : ps->piece_begin[b];
      const int np = RANKS ? src.n : ps->piece_begin[b + 1] - pb;
      float m = -INFINITY, tot = 0.f;
      for (int s0 = 0; s0 < np; s0 += kPieceBatch) {
        float lv[kPieceBatch];
        float4 v[kPieceBatch][4];
#pragma unroll
        for (int u = 0; u < kPieceBatch; ++u) {
          const int s = s0 + u;
          lv[u] = -INFINITY;
#pragma unroll
          for (int k = 0; k < 4; ++k) v[u][k] = make_float4(0.f, 0.f, 0.f, 0.f);
          if (s < np) {
            const float* sp;
            if (RANKS) {
              lv[u] = src.lse[s][trow];
              sp = src.o[s] + trow * a.d_c + 8 * gc;
            } else {
              const size_t pr = (size_t)(pb + s) * rows_total + row;
              lv[u] = a.part_lse[pr];
              sp = a.part_o + pr * a.d_c + 8 * gc;
            }
#pragma unroll
            for (int half = 0; half < 2; ++half) {
              if (cols[half]) {
                v[u][2 * half] = __ldcs(reinterpret_cast<const float4*>(sp + 256 * half));
                v[u][2 * half + 1] = __ldcs(reinterpret_cast<const float4*>(sp + 256 * half + 4));
              }
            }
          }
        }
        float mb = m;
#pragma unroll
        for (int u = 0; u < kPieceBatch; ++u) mb = fmaxf(mb, lv[u]);
        if (mb == -INFINITY) continue;                // nothing attended so far
        const float sc = (m == -INFINITY) ? 0.f : expf(m - mb);
        tot *= sc;
#pragma unroll
        for (int e = 0; e < 16; ++e) acc[e] *= sc;
#pragma unroll
        for (int u = 0; u < kPieceBatch; ++u) {
          const float wu = (lv[u] == -INFINITY) ? 0.f : expf(lv[u] - mb);
          tot += wu;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            acc[4 * k + 0] += wu * v[u][k].x;
            acc[4 * k + 1] += wu * v[u][k].y;
            acc[4 * k + 2] += wu * v[u][k].z;
            acc[4 * k + 3] += wu * v[u][k].w;
          }
        }
        m = mb;
      }
      const float lse_all = (m == -INFINITY) ? -INFINITY : m + logf(tot);
      const float inv = (m == -INFINITY) ? 0.f : 1.f / tot;
#pragma unroll
      for (int e = 0; e < 16; ++e) acc[e] *= inv;
      if (gc == 0 && a.lse != nullptr) a.lse[trow] = lse_all;
      if (lat_mode) {
        // this rank's merged latent output, for the rank merge
        float* dst = a.out_lat + trow * a.d_c + 8 * gc;
#pragma unroll
        for (int half = 0; half < 2; ++half)
          if (cols[half]) {
            *reinterpret_cast<float4*>(dst + 256 * half) =
                make_float4(acc[8 * half], acc[8 * half + 1], acc[8 * half + 2], acc[8 * half + 3]);
            *reinterpret_cast<float4*>(dst + 256 * half + 4) =
                make_float4(acc[8 * half + 4], acc[8 * half + 5], acc[8 * half + 6], acc[8 * half + 7]);
          }
      }
    }
    if (lat_mode) return;
    // rows of tokens past T and columns past d_c hold zeros
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      uint32_t hi[4], lo[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float x0 = acc[8 * half + 2 * e], x1 = acc[8 * half + 2 * e + 1];
        hi[e] = pack_bf16x2(x0, x1);
        lo[e] = pack_bf16x2(x0 - bf16_lo(hi[e]), x1 - bf16_hi(hi[e]));
      }
      const int cc8 = 32 * half + gc;                  // 16-byte chunk of the row
      const uint32_t blk = o_s + (cc8 >> 3) * kOBlock;
      asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(blk + swz(j, cc8 & 7)), "r"(hi[0]),
                   "r"(hi[1]), "r"(hi[2]), "r"(hi[3]) : "memory");
      asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(blk + swz(kTok + j, cc8 & 7)), "r"(lo[0]),
                   "r"(lo[1]), "r"(lo[2]), "r"(lo[3]) : "memory");
    }
  }
  asm volatile("cp.async.wait_all;" ::: "memory");
  fence_proxy_async_smem();   // operands written by this thread -> the tensor core
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  // 2. per chunk of 128 out rows: one thread issues the MMA chain over the latent
  //    columns; warps 0-3 read D (lane = out row, columns = hi and lo of each
  //    token) and store hi + lo
  const uint32_t idesc = idesc_bf16_f32(128, 2 * kTok, 0, 0);
  const int ksteps = (ncol + 15) / 16;
  bool ok = true;
  for (int v0 = 0, chunk = 0; v0 < a.v_head; v0 += kVChunk, ++chunk) {
    if (v0 > 0) {
      stage_w(v0);
      asm volatile("cp.async.wait_all;" ::: "memory");
      fence_proxy_async_smem();
      tc_fence_before();
      __syncthreads();
      tc_fence_after();
    }
    if (warp == 0) {
      if (elect_lane()) {
        for (int ks = 0; ks < ksteps; ++ks) {
          const uint32_t kb = ks >> 2, k4 = ks & 3;
          const uint64_t da = smem_desc(w_s + kb * kWBlock + k4 * 32, 16, 1024, kSwizzle128);
          const uint64_t db = smem_desc(o_s + kb * kOBlock + k4 * 32, 16, 1024, kSwizzle128);
          mma_bf16(tmem, da, db, idesc, ks > 0 ? 1u : 0u);
        }
        mma_commit(mma_bar);
      }
      __syncwarp();
    }
    if (warp < 4) {
      // D complete: a bounded wait (the MMAs of this CTA only)
      ok = mbar_wait_drain(mma_bar, chunk & 1, 1ll << 31);
      if (!ok && lane == 0) record_status(a.dev_status, MLA_ERR_TIMEOUT);
      tc_fence_after();
      float dv[32];
      tmem_ld32(tmem + (uint32_t(warp * 32) << 16), dv);
      tmem_wait_ld();
      const int v = v0 + warp * 32 + lane;
      if (ok && v < a.v_head) {
#pragma unroll
        for (int tl = 0; tl < kTok; ++tl) {
          const int t = t0 + tl;
          if (t < T) a.out[((size_t)t * a.n_heads + h) * a.v_head + v] = f32_to_bf16(dv[tl] + dv[kTok + tl]);
        }
      }
    }
    tc_fence_before();
    __syncthreads();   // D read and the A operand free before the next chunk's MMAs
    tc_fence_after();
  }
  if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace

size_t decode_combine_smem_bytes(int d_c) {
  (void)d_c;
  return 1024 + (size_t)kKBlocks * (kWBlock + kOBlock) + ((sizeof(PlanSmem) + 15) & ~size_t(15)) + 64;
}

namespace {

template <bool RANKS>
cudaError_t launch_combine_impl(const DecodeArgs& a, const RankSources& src, cudaStream_t stream) {
  const size_t smem = decode_combine_smem_bytes(a.d_c);
  cudaError_t e = cudaFuncSetAttribute(decode_combine_kernel<RANKS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  const int T = a.batch * a.nq;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.n_heads, (T + kTok - 1) / kTok, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1] = {pdl_attribute()};
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, decode_combine_kernel<RANKS>, a, src);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode_combine(const DecodeArgs& a, cudaStream_t stream) {
  RankSources none = {};
  return launch_combine_impl<false>(a, none, stream);
}

cudaError_t launch_merge_ranks(const DecodeArgs& a, const RankSources& src, cudaStream_t stream) {
  return launch_combine_impl<true>(a, src, stream);
}

}  // namespace mla
