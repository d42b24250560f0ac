// Combine of the split-KV partials, then the W_UV up-projection.
//
// For query row (token t, head h) with pieces s of its sequence:
//   LSE   = ln sum_s exp(lse_s)
//   o_lat = sum_s exp(lse_s - LSE) * O_s          (O_s already normalised per piece)
//   out[t][h][v] = sum_c W_UV[h][v][c] * o_lat[c]  (values up-projected once, after
//                                                   attending over latents)
// Work split: one CTA per (head, group of 16 query tokens) over all d_c latent
// columns.  Its 512 threads merge the partials (32 per token, each owning 16
// columns; each partial byte is read once, by one CTA), then 16 warps multiply
// the merged rows by W_UV,h on the tensor cores (mma.sync, fp32 accumulate,
// o_lat split into two bf16 terms, hi + lo, which keeps about 16 bits of its
// mantissa): warp w takes out rows [16 (w mod 8), +16) and half of the latent
// columns, the two halves summed in shared memory.  Independent accumulators
// (hi and lo terms, even and odd k slices) keep each mma.sync dependence chain
// 8 deep.  W_UV,h (a chunk of 128 out rows) is staged in shared memory by
// cp.async before the kernel waits for the split kernel's partials, so after
// that wait only the merge, the products and the stores remain.
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

namespace mla {

namespace {

constexpr int kThreads = 512;
constexpr int kTok = 16;       // query tokens per CTA
constexpr int kCols = 512;     // latent columns per CTA (d_c <= 512)
constexpr int kVChunk = 128;   // out rows per round (8 row tiles x 16)
constexpr int kOStride = kCols + 8;    // bf16 row stride of the merged rows (16-byte pad)
constexpr int kWStride = kCols + 8;    // bf16 row stride of the staged W_UV rows (16-byte pad)
constexpr int kPieceBatch = 4;         // pieces whose loads are in flight at once

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

template <bool RANKS>
__global__ void __launch_bounds__(kThreads, 1)
decode_combine_kernel(DecodeArgs a, const __grid_constant__ RankSources src) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  PlanSmem* ps = reinterpret_cast<PlanSmem*>(smem_raw);
  uint16_t* o_hi = reinterpret_cast<uint16_t*>(smem_raw + ((sizeof(PlanSmem) + 15) & ~size_t(15)));
  uint16_t* o_lo = o_hi + kTok * kOStride;
  float* red = reinterpret_cast<float*>(o_lo + kTok * kOStride);       // [kVChunk][kTok] upper-half products
  uint16_t* wsm = reinterpret_cast<uint16_t*>(red + kVChunk * kTok);  // [kVChunk][kWStride] W_UV rows

  const int h = blockIdx.x;
  const int t0 = blockIdx.y * kTok;
  const int T = a.batch * a.nq;
  const int rows_total = a.nq * a.n_heads;
  const int ncol = a.d_c;                       // multiple of 8, <= kCols
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, q = lane & 3;
  const uint16_t* wh = a.w_uv + (size_t)h * a.v_head * a.d_c;
  // W_UV,h rows [v0, v0 + kVChunk) -> shared memory (zeros outside the matrix)
  auto stage_w = [&](int v0) {
    for (int idx = tid; idx < kVChunk * (kCols / 8); idx += kThreads) {
      const int vl = idx / (kCols / 8), cc = 8 * (idx % (kCols / 8));
      uint16_t* dst = wsm + vl * kWStride + cc;
      if (v0 + vl < a.v_head && cc < ncol) {
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(dst)),
                     "l"(wh + (size_t)(v0 + vl) * a.d_c + cc)
                     : "memory");
      } else {
        *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
      }
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };

  const bool lat_mode = !RANKS && a.out_lat != nullptr;
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
      const int c0 = 256 * half + 8 * gc;
      *reinterpret_cast<uint4*>(o_hi + j * kOStride + c0) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
      *reinterpret_cast<uint4*>(o_lo + j * kOStride + c0) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
    }
  }
  asm volatile("cp.async.wait_all;" ::: "memory");
  __syncthreads();

  // 2. per chunk of 128 out rows: warp w multiplies its 16 rows of W_UV by the
  //    merged rows over latent half w / 8 (32-wide k slices, see mma_frag.cuh);
  //    the upper half's products go through shared memory to the lower half's
  //    warp, which adds them and stores out
  const int rt = warp & 7, kh = warp >> 3;
  for (int v0 = 0; v0 < a.v_head; v0 += kVChunk) {
    if (v0 > 0) {
      __syncthreads();   // every warp is done with the previous chunk's W rows and products
      stage_w(v0);
      asm volatile("cp.async.wait_all;" ::: "memory");
      __syncthreads();
    }
    float d[2][2][2][4];   // [token tile][hi, lo term][k slice parity][fragment]
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int tm = 0; tm < 2; ++tm)
#pragma unroll
        for (int pa = 0; pa < 2; ++pa)
#pragma unroll
          for (int e = 0; e < 4; ++e) d[nt][tm][pa][e] = 0.f;
    const int va = rt * 16 + g, vb = va + 8;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int k0 = 256 * kh + 32 * u;
      if (k0 >= ncol) break;                    // the same in every lane of the warp
      const int kk = k0 + 8 * q;
      const uint4 wa = *reinterpret_cast<const uint4*>(wsm + va * kWStride + kk);
      const uint4 wb = *reinterpret_cast<const uint4*>(wsm + vb * kWStride + kk);
      const uint4 h0 = *reinterpret_cast<const uint4*>(o_hi + g * kOStride + kk);
      const uint4 l0 = *reinterpret_cast<const uint4*>(o_lo + g * kOStride + kk);
      const uint4 h1 = *reinterpret_cast<const uint4*>(o_hi + (g + 8) * kOStride + kk);
      const uint4 l1 = *reinterpret_cast<const uint4*>(o_lo + (g + 8) * kOStride + kk);
      mma_k32(d[0][0][u & 1], wa, wb, h0);
      mma_k32(d[0][1][u & 1], wa, wb, l0);
      mma_k32(d[1][0][u & 1], wa, wb, h1);
      mma_k32(d[1][1][u & 1], wa, wb, l1);
    }
    // D fragment: (row g | g+8, token column 2q | 2q+1) of each 8-token tile
    float dd[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e)
        dd[nt][e] = (d[nt][0][0][e] + d[nt][0][1][e]) + (d[nt][1][0][e] + d[nt][1][1][e]);
    if (kh == 1) {
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e)
          red[(rt * 16 + g + ((e & 2) ? 8 : 0)) * kTok + nt * 8 + 2 * q + (e & 1)] = dd[nt][e];
    }
    __syncthreads();
    if (kh == 0) {
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int vl = rt * 16 + g + ((e & 2) ? 8 : 0);
          const int tl = nt * 8 + 2 * q + (e & 1);
          const int v = v0 + vl, t = t0 + tl;
          if (v < a.v_head && t < T)
            a.out[((size_t)t * a.n_heads + h) * a.v_head + v] = f32_to_bf16(dd[nt][e] + red[vl * kTok + tl]);
        }
    }
  }
}

}  // namespace

size_t decode_combine_smem_bytes(int d_c) {
  (void)d_c;
  return ((sizeof(PlanSmem) + 15) & ~size_t(15)) + 2ull * kTok * kOStride * 2 + (size_t)kVChunk * kTok * 4 +
         (size_t)kVChunk * kWStride * 2;
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
