// Layer output projection of the decode step: y[t] = W_O concat_h(o[t, h]).
//
// Sources (page title, section): "Deep-Dive: Multi-Head Latent Attention (MLA)
// and Low-Rank KV Cache Compression in DeepSeek-V3", sec. 3 (out_proj: one
// bias-free linear map from the head-major concatenation of the heads' outputs,
// H * d_v wide, to d_model); "mla-from-scratch" README, "Absorption, and why RoPE
// breaks it" (W_UV is applied once after attending over the latents, next to W_O).
//
// With a decode step's few tokens (T = batch * nq, 16 in the V3-shaped workload)
// the product is a stream of W_O (d_model x H * d_v bf16, 235 MB at V3 shapes)
// against a small activation block that stays in L2: HBM-bound, 2 * T flops per
// weight element.  Tensor cores are used through warp-level mma.sync tiles
// because T is far below the 128-row minimum of a tcgen05 tile; what sets the
// speed is keeping enough weight bytes in flight, not the MMA rate.
//
// CTA = 4 warps on one 16-row tile of W_O (16 outputs) and 8 * NT tokens.  The
// reduction index k = h * d_v + j is cut into 32-wide slices dealt round-robin to
// the warps; each thread loads its 16-byte pieces of two weight rows and of NT
// token rows per slice (fragment convention of mma_frag.cuh), kUnroll slices at
// a time, so that every warp keeps several KB of weight loads in flight.  The
// four warps' partial tiles are summed in shared memory and rounded to bf16 once.
// The grid (d_model / 16 tiles) is small enough that all CTAs are resident at
// once (448 CTAs at V3 shapes, up to 4 per SM), so that the weight stream is
// spread over every SM for the whole launch.
#include "../../include/mla.h"
#include "common.cuh"
#include "decode.h"
#include "mma_frag.cuh"

namespace mla {

namespace {

constexpr int kOpWarps = 4;
constexpr int kOpThreads = kOpWarps * 32;
constexpr int kOpRows = 16;  // outputs (rows of W_O) per CTA

template <int NT>
struct OpUnroll {
  static constexpr int value = NT <= 2 ? 4 : 2;  // slices in flight per warp (register budget)
};

// NT: n8 token tiles per CTA (8 * NT tokens)
template <int NT>
__global__ void __launch_bounds__(kOpThreads, 4) out_proj_kernel(const OutProjArgs a) {
  constexpr int U = OpUnroll<NT>::value;
  __shared__ float red[kOpWarps][32][NT * 4];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, q = lane & 3;
  const int r0 = blockIdx.x * kOpRows;
  const int t0 = blockIdx.y * 8 * NT;
  const int K = a.K;
  const int nslices = (K + 31) / 32;
  // rows g and g + 8 of the tile; rows past d_model read row 0 and are masked
  const bool ra_ok = r0 + g < a.D, rb_ok = r0 + g + 8 < a.D;
  const uint16_t* wa = a.w_o + (size_t)(ra_ok ? r0 + g : 0) * K + 8 * q;
  const uint16_t* wb = a.w_o + (size_t)(rb_ok ? r0 + g + 8 : 0) * K + 8 * q;
  const uint16_t* xr[NT];
  bool x_ok[NT];
#pragma unroll
  for (int j = 0; j < NT; ++j) {
    const int tok = t0 + 8 * j + g;
    x_ok[j] = tok < a.T;
    xr[j] = a.x + (size_t)(x_ok[j] ? tok : 0) * K + 8 * q;
  }
  float acc[NT][4];
#pragma unroll
  for (int j = 0; j < NT; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;

  allow_dependent_launch();
  grid_dependency_wait();  // o is written by the preceding kernel

  const uint4 zero = make_uint4(0, 0, 0, 0);
  for (int s0 = warp; s0 < nslices; s0 += kOpWarps * U) {
    uint4 a0[U], a1[U], b[U][NT];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int s = s0 + u * kOpWarps;
      const int k = 32 * s;
      // K is a multiple of 8: a thread's 8-element piece is wholly inside or outside
      const bool k_ok = s < nslices && k + 8 * q < K;
      a0[u] = (k_ok && ra_ok) ? ldg_stream(wa + k) : zero;
      a1[u] = (k_ok && rb_ok) ? ldg_stream(wb + k) : zero;
#pragma unroll
      for (int j = 0; j < NT; ++j)
        b[u][j] = (k_ok && x_ok[j]) ? __ldg(reinterpret_cast<const uint4*>(xr[j] + k)) : zero;
    }
#pragma unroll
    for (int u = 0; u < U; ++u)
#pragma unroll
      for (int j = 0; j < NT; ++j) mma_k32(acc[j], a0[u], a1[u], b[u][j]);
  }

#pragma unroll
  for (int j = 0; j < NT; ++j)
#pragma unroll
    for (int c = 0; c < 4; ++c) red[warp][lane][4 * j + c] = acc[j][c];
  __syncthreads();
  // element e of a lane's fragment: token tile j = e / 4; c = e % 4 gives row
  // g (+8 for c >= 2) and token 2q (+1 for odd c) of the 16 x 8 tile
  for (int i = threadIdx.x; i < 32 * NT * 4; i += kOpThreads) {
    const int e = i / 32, ln = i % 32;
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < kOpWarps; ++w) v += red[w][ln][e];
    const int row = r0 + (ln >> 2) + ((e & 2) ? 8 : 0);
    const int tok = t0 + 8 * (e >> 2) + 2 * (ln & 3) + (e & 1);
    if (row < a.D && tok < a.T) a.y[(size_t)tok * a.D + row] = f32_to_bf16(v);
  }
}

template <int NT>
cudaError_t launch_nt(const OutProjArgs& a, cudaStream_t stream) {
  cudaLaunchAttribute attr[1] = {pdl_attribute()};
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((a.D + kOpRows - 1) / kOpRows, (a.T + 8 * NT - 1) / (8 * NT), 1);
  cfg.blockDim = dim3(kOpThreads, 1, 1);
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, out_proj_kernel<NT>, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_out_proj(const OutProjArgs& a, cudaStream_t stream) {
  if (a.T <= 8) return launch_nt<1>(a, stream);
  if (a.T <= 16) return launch_nt<2>(a, stream);
  return launch_nt<4>(a, stream);  // 32 tokens per CTA row of the grid
}

}  // namespace mla
