// Combine of the split-KV partials, then the W_UV up-projection.
//
// For query row (token t, head h) with pieces s of its sequence:
//   LSE   = ln sum_s exp(lse_s)
//   o_lat = sum_s exp(lse_s - LSE) * O_s          (O_s already normalised per piece)
//   out[t][h][v] = sum_c W_UV[h][v][c] * o_lat[c]  (values up-projected once, after
//                                                   attending over latents)
// One CTA = one head and up to 16 query tokens.  The merge runs on all 256
// threads (coalesced reads of the partials); the up-projection is a
// [v_head x d_c] x [d_c x 16] product on the tensor cores (mma.sync, fp32
// accumulate) with o_lat split into two bf16 terms (hi + lo), which keeps about
// 16 bits of its mantissa.  W_UV,h is streamed once per group of 16 tokens.
#include "common.cuh"
#include "decode.h"
#include "mma_frag.cuh"
#include "plan.cuh"

namespace mla {

namespace {

constexpr int kThreads = 256;
constexpr int kTok = 16;

__device__ __forceinline__ uint4 ld_nc_v4(const uint16_t* p) { return ldg_stream(p); }

__global__ void __launch_bounds__(kThreads)
decode_combine_kernel(DecodeArgs a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  PlanSmem* ps = reinterpret_cast<PlanSmem*>(smem_raw);
  const int kpad = ((a.d_c + 31) & ~31);                 // reduction length padded to 32
  const int ostride = kpad + 8;                          // bf16 row stride (16-byte pad: no bank conflicts)
  uint16_t* o_hi = reinterpret_cast<uint16_t*>(smem_raw + ((sizeof(PlanSmem) + 15) & ~size_t(15)));
  uint16_t* o_lo = o_hi + kTok * ostride;

  build_plan(ps, a.seq_lens, a.batch, a.nq, a.max_pages, a.page_size, a.G, nullptr);
  const int h = blockIdx.x;
  const int t0 = blockIdx.y * kTok;
  const int T = a.batch * a.nq;
  const int rows_total = a.nq * a.n_heads;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  // 1. merge: 16 threads per token, each owning 8 consecutive columns per 128
  {
    const int j = tid >> 4, sub = tid & 15;
    const int t = t0 + j;
    float lse_all = -INFINITY;
    int pb = 0, np = 0, row = 0;
    if (t < T) {
      const int b = t / a.nq, i = t % a.nq;
      row = i * a.n_heads + h;
      pb = ps->piece_begin[b];
      np = ps->piece_begin[b + 1] - pb;
      float mx = -INFINITY;
      for (int s = 0; s < np; ++s) mx = fmaxf(mx, a.part_lse[(size_t)(pb + s) * rows_total + row]);
      if (mx != -INFINITY) {
        float tot = 0.f;
        for (int s = 0; s < np; ++s) {
          const float l = a.part_lse[(size_t)(pb + s) * rows_total + row];
          tot += (l == -INFINITY) ? 0.f : expf(l - mx);
        }
        lse_all = mx + logf(tot);
      }
      if (sub == 0 && a.lse != nullptr) a.lse[(size_t)t * a.n_heads + h] = lse_all;
    }
    for (int c0 = sub * 8; c0 < kpad; c0 += 128) {
      float acc[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] = 0.f;
      if (lse_all != -INFINITY && c0 < a.d_c) {
        for (int s0 = 0; s0 < np; s0 += 4) {         // four pieces' loads in flight at once
          float4 v0[4], v1[4];
          float wgt[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int s = s0 + u;
            wgt[u] = 0.f;
            v0[u] = v1[u] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (s < np) {
              const float l = a.part_lse[(size_t)(pb + s) * rows_total + row];
              const float* src = a.part_o + ((size_t)(pb + s) * rows_total + row) * a.d_c + c0;
              v0[u] = *reinterpret_cast<const float4*>(src);
              v1[u] = *reinterpret_cast<const float4*>(src + 4);
              wgt[u] = (l == -INFINITY) ? 0.f : expf(l - lse_all);
            }
          }
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            acc[0] += wgt[u] * v0[u].x; acc[1] += wgt[u] * v0[u].y;
            acc[2] += wgt[u] * v0[u].z; acc[3] += wgt[u] * v0[u].w;
            acc[4] += wgt[u] * v1[u].x; acc[5] += wgt[u] * v1[u].y;
            acc[6] += wgt[u] * v1[u].z; acc[7] += wgt[u] * v1[u].w;
          }
        }
      }
      uint32_t hi[4], lo[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float x0 = acc[2 * e], x1 = acc[2 * e + 1];
        hi[e] = pack_bf16x2(x0, x1);
        lo[e] = pack_bf16x2(x0 - bf16_lo(hi[e]), x1 - bf16_hi(hi[e]));
      }
      *reinterpret_cast<uint4*>(o_hi + j * ostride + c0) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
      *reinterpret_cast<uint4*>(o_lo + j * ostride + c0) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
    }
  }
  __syncthreads();

  // 2. out[t][v] = sum_c W_UV,h[v][c] o_lat[t][c]: warp per 16 value rows,
  //    two 8-token tiles, reduction in 32-wide slices (see mma_frag.cuh)
  const int g = lane >> 2, q = lane & 3;
  const uint16_t* wh = a.w_uv + (size_t)h * a.v_head * a.d_c;
  for (int m0 = warp * 16; m0 < a.v_head; m0 += 8 * 16) {
    float d0[4] = {0.f, 0.f, 0.f, 0.f}, d1[4] = {0.f, 0.f, 0.f, 0.f};
    const int va = m0 + g, vb = m0 + g + 8;
    for (int kb = 0; kb < kpad; kb += 128) {          // four 32-wide slices' weights in flight at once
      uint4 ra[4], rb[4];
      const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int kk = kb + 32 * u + 8 * q;
        const bool kin = kk < a.d_c;
        ra[u] = (kin && va < a.v_head) ? ld_nc_v4(wh + (size_t)va * a.d_c + kk) : z;
        rb[u] = (kin && vb < a.v_head) ? ld_nc_v4(wh + (size_t)vb * a.d_c + kk) : z;
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int kk = kb + 32 * u + 8 * q;
        if (kk >= kpad) break;
        const uint4 h0 = *reinterpret_cast<const uint4*>(o_hi + g * ostride + kk);
        const uint4 l0 = *reinterpret_cast<const uint4*>(o_lo + g * ostride + kk);
        const uint4 h1 = *reinterpret_cast<const uint4*>(o_hi + (g + 8) * ostride + kk);
        const uint4 l1 = *reinterpret_cast<const uint4*>(o_lo + (g + 8) * ostride + kk);
        mma_k32(d0, ra[u], rb[u], h0);
        mma_k32(d0, ra[u], rb[u], l0);
        mma_k32(d1, ra[u], rb[u], h1);
        mma_k32(d1, ra[u], rb[u], l1);
      }
    }
    // D fragment: (row g | g+8, token column 2q | 2q+1) of each 8-token tile
    const float* dd[2] = {d0, d1};
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int v = m0 + g + ((e & 2) ? 8 : 0);
        const int t = t0 + nt * 8 + 2 * q + (e & 1);
        if (v < a.v_head && t < T) a.out[((size_t)t * a.n_heads + h) * a.v_head + v] = f32_to_bf16(dd[nt][e]);
      }
    }
  }
}

}  // namespace

size_t decode_combine_smem_bytes(int d_c) {
  const int kpad = ((d_c + 31) & ~31);
  return ((sizeof(PlanSmem) + 15) & ~size_t(15)) + 2ull * kTok * (kpad + 8) * 2;
}

cudaError_t launch_decode_combine(const DecodeArgs& a, cudaStream_t stream) {
  const size_t smem = decode_combine_smem_bytes(a.d_c);
  cudaError_t e = cudaFuncSetAttribute(decode_combine_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int T = a.batch * a.nq;
  dim3 grid(a.n_heads, (T + kTok - 1) / kTok);
  decode_combine_kernel<<<grid, kThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace mla
