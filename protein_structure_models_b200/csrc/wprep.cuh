// wprep.cuh -- the output-weight preparation, run by CTAs of the prologue's
// launch (it depends only on w_out, so it overlaps the lift).
#pragma once
#include "kernels.h"
#include "sm100.cuh"

namespace fipa {

// w_out [F, Cout] -> wT [Cout_pad, Kgp] fp16, K-major, in the head-block order
// of the projection operand (plan.h): column k = (h * nseg + seg) * Wh8 + j
// holds row f(h, j) of w_out, f the page's head-major feature index:
//   j <  Dv           scalar   f = h*Dv + j
//   j <  Dv + 4Q      x,y,z,len  f = H*Dv + blk*H*Q + h*Q + q   (j = Dv + blk*Q + q)
//   j <  Dv + 4Q + Cz pair     f = H*Dv + 4*H*Q + h*Cz + c
// and zero for the padding j >= Wh and k >= Kg.  Segments:
//   bf16 inputs: [ w | w ]            (w is exact in fp16)
//   f32  inputs: [ w hi | w lo | w hi ]
// 32 x 32 tiles over (f, n) transposed through shared memory (coalesced reads);
// one tile per call, 256 threads (32 x 8).
__device__ __forceinline__ int feature_block_col(const Plan& p, int f, int* h) {
  const int HDv = p.H * p.Dv, HQ = p.H * p.Q;
  if (f < HDv) { *h = f / p.Dv; return f - *h * p.Dv; }
  if (f < HDv + 4 * HQ) {
    const int g = f - HDv, blk = g / HQ, rem = g - blk * HQ;
    *h = rem / p.Q;
    return p.Dv + blk * p.Q + (rem - *h * p.Q);
  }
  const int g = f - HDv - 4 * HQ;
  *h = g / p.Cz;
  return p.Dv + 4 * p.Q + (g - *h * p.Cz);
}

template <typename T>
__device__ __forceinline__ void weight_prep_tile(const Plan& p, const T* w, __half* wT, int cout_pad, int bx, int by,
                                                 float (*tile)[33]) {
  const int f0 = bx * 32, n0 = by * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  for (int k = ty; k < 32; k += 8) {
    const int f = f0 + k, n = n0 + tx;
    tile[k][tx] = (f < p.F && n < p.Cout) ? ld_in(w, (size_t)f * p.Cout + n) : 0.f;
  }
  __syncthreads();
  const int f = f0 + tx;
  int h = 0;
  const int j = f < p.F ? feature_block_col(p, f, &h) : 0;
  for (int k = ty; k < 32; k += 8) {
    const int n = n0 + k;
    if (n >= cout_pad || f >= p.F) continue;
    const float v = tile[tx][k];
    const __half hi = __float2half_rn(v), lo = __float2half_rn(v - __half2float(hi));
    __half* row = wT + (size_t)n * p.Kgp + (size_t)h * p.nseg * p.Wh8 + j;
    for (int seg = 0; seg < p.nseg; ++seg) row[seg * p.Wh8] = (p.f32 && seg == 1) ? lo : hi;
  }
  if (bx == 0) {
    // padding columns: j in [Wh, Wh8) of every head segment, and [Kg, Kgp)
    const int padw = p.Wh8 - p.Wh, nblk = p.H * p.nseg;
    for (int k = ty; k < 32; k += 8) {
      const int n = n0 + k;
      if (n >= cout_pad) continue;
      __half* row = wT + (size_t)n * p.Kgp;
      for (int e = tx; e < nblk * padw; e += 32) {
        const int bk = e / padw;
        row[(size_t)bk * p.Wh8 + p.Wh + (e - bk * padw)] = __float2half_rn(0.f);
      }
      for (int c = p.Kg + tx; c < p.Kgp; c += 32) row[c] = __float2half_rn(0.f);
    }
  }
}

}  // namespace fipa
