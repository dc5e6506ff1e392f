// prologue.cu -- frames to global points and the lifted Q / K / V rows (HBM-bound).
//
// Two kernels:
//   origin: one CTA per (128-residue tile, sample) reduces the origin o_G of
//           each 32-residue group (mean translation of its valid residues) and
//           the tile's valid flag;
//   lift:   one CTA per 8 residues of a sample, all heads.  It stages the
//           frames, z1 rows and Wb^T in shared memory, applies every frame
//           T_i(x) = R_i x + t_i (page "Invariant point attention (IPA)",
//           Required behavior: column-vector convention) to all query / key /
//           value points in parallel, and then writes every lifted row of
//           plan.h as 16-byte chunks of 8 fp16 values.  Each column segment is
//           padded to a multiple of 8, so a chunk never straddles two segments.
// The distance weight g is folded into the query point columns, following the
// squared-norm expansion of FlashIPA's lifted attention.
#include "kernels.h"
#include "sm100.cuh"

namespace fipa {
namespace {

constexpr int kLiftRes = 8;        // residues per lift CTA (divides the 128-residue tile)
constexpr int kLiftThreads = 256;

__device__ __forceinline__ __half hi_half(float x) { return __float2half_rn(x); }
__device__ __forceinline__ __half lo_half(float x) {
  return __float2half_rn(x - __half2float(__float2half_rn(x)));
}
__device__ __forceinline__ uint32_t pack2(float a, float b, bool lo) {
  const __half x = lo ? lo_half(a) : hi_half(a), y = lo ? lo_half(b) : hi_half(b);
  return (uint32_t)__half_as_ushort(x) | ((uint32_t)__half_as_ushort(y) << 16);
}
__device__ __forceinline__ void store8(__half* dst, const float (&v)[8], bool lo) {
  uint4 u;
  u.x = pack2(v[0], v[1], lo);
  u.y = pack2(v[2], v[3], lo);
  u.z = pack2(v[4], v[5], lo);
  u.w = pack2(v[6], v[7], lo);
  *reinterpret_cast<uint4*>(dst) = u;
}

struct PrologueArgs {
  Plan p;
  Inputs in;
  Work w;
};

template <typename T>
__global__ void __launch_bounds__(kTile) fipa_origin_kernel(const PrologueArgs a) {
  // warp w reduces 32-residue group 4t+w of the 128-residue tile t
  const Plan& p = a.p;
  const T* tr = static_cast<const T*>(a.in.trans);
  const int t = blockIdx.x, b = blockIdx.y, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  __shared__ int s_any[kTile / 32];
  float sx = 0.f, sy = 0.f, sz = 0.f, cnt = 0.f;
  const int i = t * kTile + threadIdx.x;
  if (i < p.N && a.in.mask[(size_t)b * p.N + i]) {
    const size_t o = ((size_t)b * p.N + i) * 3;
    sx = ld_in(tr, o + 0); sy = ld_in(tr, o + 1); sz = ld_in(tr, o + 2); cnt = 1.f;
  }
  for (int off = 16; off; off >>= 1) {
    sx += __shfl_xor_sync(0xffffffffu, sx, off);
    sy += __shfl_xor_sync(0xffffffffu, sy, off);
    sz += __shfl_xor_sync(0xffffffffu, sz, off);
    cnt += __shfl_xor_sync(0xffffffffu, cnt, off);
  }
  if (lane == 0) {
    const float inv = cnt > 0.f ? 1.f / cnt : 0.f;
    a.w.orig[(size_t)b * p.nG + t * 4 + warp] = make_float4(sx * inv, sy * inv, sz * inv, cnt);
    s_any[warp] = cnt > 0.f;
  }
  __syncthreads();
  if (threadIdx.x == 0) a.w.flag[(size_t)b * p.nT + t] = (s_any[0] | s_any[1] | s_any[2] | s_any[3]) ? 1 : 0;
}

template <typename T>
__global__ void __launch_bounds__(kLiftThreads) fipa_lift_kernel(const PrologueArgs a) {
  const Plan& p = a.p;
  const T* q = static_cast<const T*>(a.in.q);
  const T* k = static_cast<const T*>(a.in.k);
  const T* v = static_cast<const T*>(a.in.v);
  const T* qp = static_cast<const T*>(a.in.q_pts);
  const T* kp = static_cast<const T*>(a.in.k_pts);
  const T* vp = static_cast<const T*>(a.in.v_pts);
  const T* rot = static_cast<const T*>(a.in.rot);
  const T* tr = static_cast<const T*>(a.in.trans);
  const T* z1 = static_cast<const T*>(a.in.z1);
  const T* z2 = static_cast<const T*>(a.in.z2);
  const T* Wb = static_cast<const T*>(a.in.Wb);
  const T* raw = static_cast<const T*>(a.in.raw);
  const int N = p.N, H = p.H, P = p.P, Q = p.Q, Cz = p.Cz, RCz = p.R * p.Cz;
  const int b = blockIdx.y, i0 = blockIdx.x * kLiftRes;
  const int nres = min(kLiftRes, N - i0);
  const int npt = 2 * P + Q;                 // query, key and value points of one head

  extern __shared__ float sh[];
  float* wbt = sh;                                   // [H][Cz]  Wb^T / sqrt(3)
  float* z1s = wbt + H * Cz;                         // [8][R*Cz]
  float* z2s = z1s + kLiftRes * RCz;                 // [8][R*Cz]
  float* pts = z2s + kLiftRes * RCz;                 // [8][H][npt][3]  global point - o_G
  float* frm = pts + kLiftRes * H * npt * 3;         // [8][12]  R (row-major), t - o_G
  float* qs = frm + kLiftRes * 12;                   // [8][H][D]
  float* ks = qs + kLiftRes * H * p.D;               // [8][H][D]
  float* vs = ks + kLiftRes * H * p.D;               // [8][H][Dv]
  __shared__ float s_gamma[64];
  __shared__ int s_valid[kLiftRes];

  // ---- stage every input of the 8 residues (independent loads, issued together)
  const float inv_sqrt3 = rsqrtf(3.0f);
  const size_t bi0 = (size_t)b * N + i0;
  for (int e = threadIdx.x; e < H * Cz; e += blockDim.x) {
    const int h = e / Cz, c = e - h * Cz;
    wbt[e] = ld_in(Wb, (size_t)c * H + h) * inv_sqrt3;
  }
#pragma unroll 4
  for (int e = threadIdx.x; e < nres * RCz; e += blockDim.x) {
    z1s[e] = ld_in(z1, bi0 * RCz + e);
    z2s[e] = ld_in(z2, bi0 * RCz + e);
  }
#pragma unroll 4
  for (int e = threadIdx.x; e < nres * H * p.D; e += blockDim.x) {
    qs[e] = ld_in(q, bi0 * H * p.D + e);
    ks[e] = ld_in(k, bi0 * H * p.D + e);
  }
#pragma unroll 4
  for (int e = threadIdx.x; e < nres * H * p.Dv; e += blockDim.x) vs[e] = ld_in(v, bi0 * H * p.Dv + e);
  for (int e = threadIdx.x; e < nres * 12; e += blockDim.x) {
    const int r = e / 12, c = e - r * 12;
    const size_t bi = bi0 + r;
    if (c < 9) {
      frm[e] = ld_in(rot, bi * 9 + c);
    } else {
      const float4 o = a.w.orig[(size_t)b * p.nG + (i0 + r) / kGroup];
      frm[e] = ld_in(tr, bi * 3 + (c - 9)) - (c == 9 ? o.x : c == 10 ? o.y : o.z);
    }
  }
  for (int h = threadIdx.x; h < H && h < 64; h += blockDim.x) s_gamma[h] = point_weight(ld_in(raw, h), P);
  if (threadIdx.x < nres) s_valid[threadIdx.x] = a.in.mask[bi0 + threadIdx.x] != 0;
  __syncthreads();

  // ---- every point of every head of the 8 residues, relative to its group origin
#pragma unroll 4
  for (int e = threadIdx.x; e < nres * H * npt; e += blockDim.x) {
    const int r = e / (H * npt), rem = e - r * H * npt, h = rem / npt, pt = rem - h * npt;
    const size_t bih = ((size_t)b * N + i0 + r) * H + h;
    const T* src = pt < P ? qp + (bih * P + pt) * 3
                 : pt < 2 * P ? kp + (bih * P + (pt - P)) * 3 : vp + (bih * Q + (pt - 2 * P)) * 3;
    const float x0 = ld_in(src, 0), x1 = ld_in(src, 1), x2 = ld_in(src, 2);
    const float* F = frm + r * 12;
    float* o = pts + (size_t)e * 3;
    o[0] = F[0] * x0 + F[1] * x1 + F[2] * x2 + F[9];
    o[1] = F[3] * x0 + F[4] * x1 + F[5] * x2 + F[10];
    o[2] = F[6] * x0 + F[7] * x1 + F[8] * x2 + F[11];
  }
  __syncthreads();

  // ---- per (residue, head) fp32 corrections (and the fp32 points of float32 mode)
  for (int e = threadIdx.x; e < nres * H; e += blockDim.x) {
    const int r = e / H, h = e - r * H;
    const float g = s_gamma[h < 64 ? h : 63];
    const float* pa = pts + (size_t)e * npt * 3;
    const float* pb = pa + 3 * P;
    float Ax = 0.f, Ay = 0.f, Az = 0.f, a2 = 0.f, Bx = 0.f, By = 0.f, Bz = 0.f, b2 = 0.f;
    for (int pp = 0; pp < P; ++pp) {
      Ax += pa[3 * pp]; Ay += pa[3 * pp + 1]; Az += pa[3 * pp + 2];
      a2 += pa[3 * pp] * pa[3 * pp] + pa[3 * pp + 1] * pa[3 * pp + 1] + pa[3 * pp + 2] * pa[3 * pp + 2];
      Bx += pb[3 * pp]; By += pb[3 * pp + 1]; Bz += pb[3 * pp + 2];
      b2 += pb[3 * pp] * pb[3 * pp] + pb[3 * pp + 1] * pb[3 * pp + 1] + pb[3 * pp + 2] * pb[3 * pp + 2];
    }
    const bool valid = s_valid[r] != 0;
    const size_t bhi = ((size_t)b * H + h) * N + i0 + r;
    if (p.geo_simt) {
      a.w.kvec[bhi] = make_float4(valid ? 0.f : -INFINITY, 0.f, 0.f, 0.f);
      a.w.qvec[bhi] = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int x = 0; x < 3 * P; ++x) {
        a.w.QP[bhi * 3 * P + x] = pa[x];
        a.w.KP[bhi * 3 * P + x] = valid ? pb[x] : 0.f;
      }
    } else {
      a.w.kvec[bhi] = valid ? make_float4(-g * b2, Bx, By, Bz) : make_float4(-INFINITY, 0.f, 0.f, 0.f);
      a.w.qvec[bhi] = make_float4(Ax, Ay, Az, -g * a2);
    }
  }

  // ---- every lifted row as 16-byte chunks (8 fp16 values of one segment):
  // one warp per row, lanes over its chunks
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarp = blockDim.x >> 5;
  const float sqk = rsqrtf(3.0f * (float)p.D);
  const int sq = p.nsq * p.D8;          // scalar columns of the query / key head part
  const int sv = p.nsv * p.Dv8;         // scalar columns of the value head part
  for (int row = warp; row < nres * H; row += nwarp) {
    const int r = row / H, h = row - r * H, i = i0 + r;
    const bool valid = s_valid[r] != 0;
    const float* qsr = qs + (r * H + h) * p.D;
    const float* ksr = ks + (r * H + h) * p.D;
    const float* vsr = vs + (r * H + h) * p.Dv;
    const float* pa = pts + ((size_t)r * H + h) * npt * 3;
    const float* pb = pa + 3 * P;
    const float* pg = pb + 3 * P;
    const float g2 = 2.f * s_gamma[h < 64 ? h : 63];
    const size_t rowid = ((size_t)b * H + h) * N + i;
    // query row: [ scalar | points (tensor-core mode) | pad ] [ pair part ]
    __half* qrow = a.w.Q + rowid * p.Kq;
    for (int c8 = lane; c8 < p.Kq / 8; c8 += 32) {
      const int col = c8 * 8;
      float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      bool lo = false;
      if (valid) {
        if (col < sq) {
          const int seg = col / p.D8, e0 = col - seg * p.D8;
          lo = (seg == 2);
#pragma unroll
          for (int t = 0; t < 8; ++t) if (e0 + t < p.D) v[t] = qsr[e0 + t] * sqk;
        } else if (col < p.KHp) {
          if (!p.geo_simt && col < sq + 3 * p.P38) {
            const int seg = (col - sq) / p.P38, e0 = col - sq - seg * p.P38;
            lo = (seg == 2);
#pragma unroll
            for (int t = 0; t < 8; ++t) if (e0 + t < 3 * P) v[t] = g2 * pa[e0 + t];
          }
        } else {
          const int cc = col - p.KHp;
          int e0;
          if (p.nqz == 2) {                        // [u hi | u lo], each Zp wide
            lo = cc >= p.Zp;
            e0 = lo ? cc - p.Zp : cc;
          } else {                                 // [u hi | u hi | u lo], RC8 apart
            const int seg = cc / p.RC8;
            e0 = seg < p.nz ? cc - seg * p.RC8 : RCz;
            lo = (seg == 2);
          }
          if (e0 < RCz) {
            int rr = e0 / Cz, c0 = e0 - rr * Cz;
#pragma unroll
            for (int t = 0; t < 8; ++t) {
              if (e0 + t < RCz) v[t] = z1s[r * RCz + e0 + t] * wbt[h * Cz + c0];
              if (++c0 == Cz) { c0 = 0; ++rr; }
            }
          }
        }
      }
      store8(qrow + col, v, lo);
    }
    // key row (head part): [ scalar | points (tensor-core mode) | pad ]
    __half* krow = a.w.KH + rowid * p.KHp;
    for (int c8 = lane; c8 < p.KHp / 8; c8 += 32) {
      const int col = c8 * 8;
      float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      bool lo = false;
      if (valid) {
        if (col < sq) {
          const int seg = col / p.D8, e0 = col - seg * p.D8;
          lo = (seg == 1);
#pragma unroll
          for (int t = 0; t < 8; ++t) if (e0 + t < p.D) v[t] = ksr[e0 + t];
        } else if (!p.geo_simt && col < sq + 3 * p.P38) {
          const int seg = (col - sq) / p.P38, e0 = col - sq - seg * p.P38;
          lo = (seg == 1);
#pragma unroll
          for (int t = 0; t < 8; ++t) if (e0 + t < 3 * P) v[t] = pb[e0 + t];
        }
      }
      store8(krow + col, v, lo);
    }
    // value row (head part): [ scalar | g' hi | g' lo | pad ]
    __half* vrow = a.w.VH + rowid * p.VHp;
    for (int c8 = lane; c8 < p.VHp / 8; c8 += 32) {
      const int col = c8 * 8;
      float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      bool lo = false;
      if (valid) {
        if (col < sv) {
          const int seg = col / p.Dv8, e0 = col - seg * p.Dv8;
          lo = (seg == 1);
#pragma unroll
          for (int t = 0; t < 8; ++t) if (e0 + t < p.Dv) v[t] = vsr[e0 + t];
        } else if (col < sv + 2 * p.Q38) {
          const int seg = (col - sv) / p.Q38, e0 = col - sv - seg * p.Q38;
          lo = (seg == 1);
#pragma unroll
          for (int t = 0; t < 8; ++t) if (e0 + t < 3 * Q) v[t] = pg[e0 + t];
        }
      }
      store8(vrow + col, v, lo);
    }
  }
  // pair factor rows z2 (shared by the heads): [ z2 segments | pad ]
  for (int r = warp; r < nres; r += nwarp) {
    const bool valid = s_valid[r] != 0;
    __half* zrow = a.w.Z + (bi0 + r) * p.Zp;
    for (int c8 = lane; c8 < p.Zp / 8; c8 += 32) {
      const int col = c8 * 8, seg = col / p.RC8, e0 = col - seg * p.RC8;
      float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      const bool lo = (seg == 1);
      if (valid && seg < p.nz) {
#pragma unroll
        for (int t = 0; t < 8; ++t) if (e0 + t < RCz) v[t] = z2s[r * RCz + e0 + t];
      }
      store8(zrow + col, v, lo);
    }
  }
}

}  // namespace

cudaError_t launch_prologue(const Plan& p, const Inputs& in, const Work& w, cudaStream_t s) {
  PrologueArgs a{p, in, w};
  dim3 g1(p.nT, p.B), g2((p.N + kLiftRes - 1) / kLiftRes, p.B);
  if (p.f32) {
    fipa_origin_kernel<float><<<g1, kTile, 0, s>>>(a);
    auto kfn = fipa_lift_kernel<float>;
    cudaError_t e = allow_max_smem(reinterpret_cast<const void*>(kfn));
    if (e != cudaSuccess) return e;
    kfn<<<g2, kLiftThreads, p.lift_smem, s>>>(a);
  } else {
    fipa_origin_kernel<__nv_bfloat16><<<g1, kTile, 0, s>>>(a);
    auto kfn = fipa_lift_kernel<__nv_bfloat16>;
    cudaError_t e = allow_max_smem(reinterpret_cast<const void*>(kfn));
    if (e != cudaSuccess) return e;
    kfn<<<g2, kLiftThreads, p.lift_smem, s>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace fipa
