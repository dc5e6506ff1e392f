// attention.cu -- optional dense attention output [B, H, N, N] (validation aid).
//
// Recomputes every logit from the same lifted operands and fp32 corrections
// the fused core uses, and normalises with the core's saved row statistics
// (running max M in log2 units, denominator l).  Entries whose key is not
// permitted (mask_i && mask_j && pair_mask_ij false, page "Invariant point
// attention (IPA)", Required behavior) and rows with an empty neighbourhood
// are written as exact zeros.  O(N^2) time and memory: never part of the
// fused forward's hot path.
#include "kernels.h"
#include "sm100.cuh"

namespace fipa {
namespace {

constexpr int kRows = 8;          // query rows per CTA (each key row read once per 8 queries)
constexpr float kLog2e = 1.4426950408889634f;

struct AttnArgs {
  Plan p;
  const __half* Q;
  const __half* KH;
  const __half* Z;
  const float4* kvec;
  const float4* qvec;
  const float4* orig;
  const float2* stats;
  const float* QP;
  const float* KP;
  const uint8_t* mask;
  const uint8_t* pair_mask;
  const void* raw;
  float* attention;
};

__global__ void __launch_bounds__(128) fipa_attention_kernel(const AttnArgs a) {
  const Plan& p = a.p;
  extern __shared__ float qs[];                 // [kRows][Kq]
  const int i0 = p.row0 + blockIdx.x * kRows, h = blockIdx.y, b = blockIdx.z;
  const int N = p.N, bh = b * p.H + h;
  const int iend = p.row1;                      // rows of the forward's range (<= N)
  const float raw = p.f32 ? static_cast<const float*>(a.raw)[h]
                          : __bfloat162float(static_cast<const __nv_bfloat16*>(a.raw)[h]);
  const float g = point_weight(raw, p.P);
  for (int e = threadIdx.x; e < kRows * p.Kq; e += blockDim.x) {
    const int rr = e / p.Kq, c = e - rr * p.Kq;
    const int i = i0 + rr;
    qs[e] = i < iend ? __half2float(a.Q[((size_t)bh * N + i) * p.Kq + c]) : 0.f;
  }
  __syncthreads();
  float M[kRows], l[kRows];
  bool live[kRows];
  float4 oq[kRows], qv[kRows];
  for (int rr = 0; rr < kRows; ++rr) {
    const int i = i0 + rr;
    live[rr] = false;
    if (i < iend) {
      const float2 st = a.stats[(size_t)bh * N + i];
      M[rr] = st.x; l[rr] = st.y;
      live[rr] = a.mask[(size_t)b * N + i] != 0 && st.y > 0.f;
      oq[rr] = a.orig[(size_t)b * p.nG + i / kGroup];
      qv[rr] = a.qvec[(size_t)bh * N + i];
    }
  }
  for (int j = threadIdx.x; j < N; j += blockDim.x) {
    const float4 kv = a.kvec[(size_t)bh * N + j];
    const float4 ok = a.orig[(size_t)b * p.nG + j / kGroup];
    float dot[kRows];
    for (int rr = 0; rr < kRows; ++rr) dot[rr] = 0.f;
    if (kv.x != -INFINITY) {
      // pair columns first, then the (larger) scalar and point columns, the
      // accumulation order of the fused core
      const __half* zrow = a.Z + ((size_t)b * N + j) * p.Zp;
      for (int c = 0; c < p.Zp; ++c) {
        const float zc = __half2float(zrow[c]);
        for (int qz = 0; qz < p.nqz; ++qz)      // every Qhat pair part (u hi, u lo) meets the same z2
          for (int rr = 0; rr < kRows; ++rr) dot[rr] = fmaf(qs[rr * p.Kq + p.KHp + qz * p.Zp + c], zc, dot[rr]);
      }
      const __half* krow = a.KH + ((size_t)bh * N + j) * p.KHp;
      for (int c = 0; c < p.KHp; ++c) {
        const float kc = __half2float(krow[c]);
        for (int rr = 0; rr < kRows; ++rr) dot[rr] = fmaf(qs[rr * p.Kq + c], kc, dot[rr]);
      }
    }
    for (int rr = 0; rr < kRows; ++rr) {
      const int i = i0 + rr;
      if (i >= iend) break;
      float att = 0.f;
      bool permitted = live[rr] && kv.x != -INFINITY;
      if (permitted && a.pair_mask != nullptr) permitted = a.pair_mask[((size_t)b * N + i) * N + j] != 0;
      if (permitted) {
        const float dx = oq[rr].x - ok.x, dy = oq[rr].y - ok.y, dz = oq[rr].z - ok.z;
        const float kterm = kv.x + 2.f * g * (dx * kv.y + dy * kv.z + dz * kv.w);
        float rc, x = dot[rr] + kterm;
        if (p.geo_simt) {
          // float32 inputs: exact fp32 squared distance, as in the fused core
          const int P3 = 3 * p.P;
          const float* ap = a.QP + ((size_t)bh * N + i) * P3;
          const float* bp = a.KP + ((size_t)bh * N + j) * P3;
          float d2 = 0.f;
          for (int e = 0; e < P3; ++e) {
            const float dd = (e % 3 == 0) ? dx : (e % 3 == 1) ? dy : dz;
            const float d = (ap[e] + dd) - bp[e];
            d2 = fmaf(d, d, d2);
          }
          x -= g * d2;
          rc = 0.f;
        } else {
          rc = -g * ((float)p.P * (dx * dx + dy * dy + dz * dz) +
                     2.f * (dx * qv[rr].x + dy * qv[rr].y + dz * qv[rr].z));
        }
        att = ex2_approx(fmaf(x, kLog2e, -(M[rr] - rc * kLog2e))) / l[rr];
      }
      a.attention[((size_t)bh * N + i) * N + j] = att;
    }
  }
}

}  // namespace

cudaError_t launch_attention_dump(const Plan& p, const Inputs& in, const Work& w, const Outputs& out,
                                  cudaStream_t s) {
  AttnArgs a{p, w.Q, w.KH, w.Z, w.kvec, w.qvec, w.orig, w.stats, w.QP, w.KP, in.mask, in.pair_mask, in.raw,
             out.attention};
  const size_t smem = (size_t)kRows * p.Kq * sizeof(float);
  cudaError_t e = allow_max_smem(reinterpret_cast<const void*>(fipa_attention_kernel));
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)((p.row1 - p.row0 + kRows - 1) / kRows), (unsigned)p.H, (unsigned)p.B);
  fipa_attention_kernel<<<grid, 128, smem, s>>>(a);
  return cudaGetLastError();
}

}  // namespace fipa
