// layer.cu -- the IPA layer around the fused core (float32), every weight
// supplied by the caller (page "Invariant point attention (IPA)", Required
// behavior: the core starts after the input projections and has no residual
// or frame update; this layer adds the plainest forms of those steps):
//   X = s @ W_in + b_in, split into q, k, v, q/k/v local points, z1, z2;
//   the fused core;  s' = s + update;
//   [b c d tx ty tz] = s' @ W_bb + b_bb,  R' = R R(1,b,c,d),  t' = R (tx,ty,tz) + t.
#include "kernels.h"

namespace fipa {
namespace {

// The eight core inputs a column of X belongs to, in order.
struct ProjOut {
  float* dst[8];
  int start[9];   // first column of each block; start[8] = Din
};

// X[m, n] = sum_k s[m, k] W[k, n] + bias[n], written into the block of column n
// (row-major [B*N, width] each).  64 x 64 output tile per CTA, 4 x 4 per thread.
__global__ void __launch_bounds__(256) layer_proj_kernel(const float* __restrict__ A, const float* __restrict__ W,
                                                         const float* __restrict__ bias, int M, int K, int Nout,
                                                         const ProjOut out) {
  __shared__ __align__(16) float As[32][68];
  __shared__ __align__(16) float Ws[32][68];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int m0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
  for (int k0 = 0; k0 < K; k0 += 32) {
    for (int e = threadIdx.x; e < 64 * 32; e += 256) {
      const int r = e >> 5, kk = e & 31;
      As[kk][r] = (m0 + r < M && k0 + kk < K) ? A[(size_t)(m0 + r) * K + k0 + kk] : 0.f;
      const int kk2 = e >> 6, c = e & 63;
      Ws[kk2][c] = (k0 + kk2 < K && n0 + c < Nout) ? W[(size_t)(k0 + kk2) * Nout + n0 + c] : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < 32; ++kk) {
      const float4 av = *reinterpret_cast<const float4*>(&As[kk][ty * 4]);
      const float4 wv = *reinterpret_cast<const float4*>(&Ws[kk][tx * 4]);
      const float aa[4] = {av.x, av.y, av.z, av.w}, ww[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(aa[i], ww[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int n = n0 + tx * 4 + j;
    if (n >= Nout) continue;
    int blk = 0;
    while (n >= out.start[blk + 1]) ++blk;
    const int w = out.start[blk + 1] - out.start[blk], c = n - out.start[blk];
    const float bn = bias[n];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int m = m0 + ty * 4 + i;
      if (m < M) out.dst[blk][(size_t)m * w + c] = acc[i][j] + bn;
    }
  }
}

// One warp per residue: s' = s + update, u = s' @ W_bb + b_bb (six dot products
// over Cs, reduced across the warp in a fixed order), the quaternion frame update.
__global__ void __launch_bounds__(256) layer_frame_kernel(const float* __restrict__ s, const float* __restrict__ upd,
                                                          const float* __restrict__ Wbb, const float* __restrict__ bbb,
                                                          const float* __restrict__ rot, const float* __restrict__ trans,
                                                          const uint8_t* __restrict__ mask, int M, int Cs,
                                                          float* __restrict__ out_s, float* __restrict__ out_rot,
                                                          float* __restrict__ out_trans) {
  const int lane = threadIdx.x & 31;
  const int m = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (m >= M) return;                                 // uniform over the warp
  float u[6] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  for (int c = lane; c < Cs; c += 32) {
    const float sn = s[(size_t)m * Cs + c] + upd[(size_t)m * Cs + c];
    out_s[(size_t)m * Cs + c] = sn;
#pragma unroll
    for (int e = 0; e < 6; ++e) u[e] = fmaf(sn, Wbb[(size_t)c * 6 + e], u[e]);
  }
#pragma unroll
  for (int e = 0; e < 6; ++e)
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) u[e] += __shfl_xor_sync(0xffffffffu, u[e], o);
  if (lane != 0) return;
  const float* R = rot + (size_t)m * 9;
  const float* t = trans + (size_t)m * 3;
  float* Ro = out_rot + (size_t)m * 9;
  float* to = out_trans + (size_t)m * 3;
  if (mask[m] == 0) {                                 // a masked residue keeps its frame
    for (int e = 0; e < 9; ++e) Ro[e] = R[e];
    for (int e = 0; e < 3; ++e) to[e] = t[e];
    return;
  }
  for (int e = 0; e < 6; ++e) u[e] += bbb[e];
  const float b = u[0], c = u[1], d = u[2];
  const float inv = rsqrtf(1.f + b * b + c * c + d * d);
  const float w = inv, x = b * inv, y = c * inv, z = d * inv;
  const float dR[9] = {w * w + x * x - y * y - z * z, 2.f * (x * y - w * z), 2.f * (x * z + w * y),
                       2.f * (x * y + w * z), w * w - x * x + y * y - z * z, 2.f * (y * z - w * x),
                       2.f * (x * z - w * y), 2.f * (y * z + w * x), w * w - x * x - y * y + z * z};
#pragma unroll
  for (int r = 0; r < 3; ++r) {
#pragma unroll
    for (int cc = 0; cc < 3; ++cc)
      Ro[3 * r + cc] = R[3 * r] * dR[cc] + R[3 * r + 1] * dR[3 + cc] + R[3 * r + 2] * dR[6 + cc];
    to[r] = R[3 * r] * u[3] + R[3 * r + 1] * u[4] + R[3 * r + 2] * u[5] + t[r];
  }
}

}  // namespace

cudaError_t launch_layer_proj(const float* s, const float* W_in, const float* b_in, int M, int Cs, int Din,
                              float* const dst[8], const int start[9], cudaStream_t st) {
  ProjOut o;
  for (int i = 0; i < 8; ++i) o.dst[i] = dst[i];
  for (int i = 0; i < 9; ++i) o.start[i] = start[i];
  layer_proj_kernel<<<dim3(cdiv(Din, 64), cdiv(M, 64)), 256, 0, st>>>(s, W_in, b_in, M, Cs, Din, o);
  return cudaGetLastError();
}

cudaError_t launch_layer_frame(const float* s, const float* upd, const float* W_bb, const float* b_bb, const float* rot,
                               const float* trans, const uint8_t* mask, int M, int Cs, float* out_s, float* out_rot,
                               float* out_trans, cudaStream_t st) {
  layer_frame_kernel<<<cdiv(M, 8), 256, 0, st>>>(s, upd, W_bb, b_bb, rot, trans, mask, M, Cs, out_s, out_rot,
                                                  out_trans);
  return cudaGetLastError();
}

}  // namespace fipa
