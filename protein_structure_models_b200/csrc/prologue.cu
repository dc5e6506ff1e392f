// prologue.cu -- frames to global points and the lifted Q / K / V rows (HBM-bound).
//
// One CTA per (128-residue tile, sample).  The CTA first reduces the tile's
// origin o_T (mean translation of its valid residues), then one warp per
// residue applies the frame T_i(x) = R_i x + t_i ("Required behavior": frames,
// column-vector convention) to every query/key/value point of every head,
// expresses the global points relative to o_T, and writes the lifted rows
// documented in plan.h, with the distance weight folded into the query
// columns (squared-norm expansion of FlashIPA's lifted attention).
#include "kernels.h"
#include "sm100.cuh"

namespace fipa {
namespace {

constexpr int kPrologueWarps = 16;

__device__ __forceinline__ __half hi_half(float x) { return __float2half_rn(x); }
__device__ __forceinline__ __half lo_half(float x) {
  return __float2half_rn(x - __half2float(__float2half_rn(x)));
}
// Part `seg` of a value stored as `pattern`: 0 -> hi, 1 -> lo.
__device__ __forceinline__ __half part(float x, int is_lo) { return is_lo ? lo_half(x) : hi_half(x); }

struct PrologueArgs {
  Plan p;
  Inputs in;
  Work w;
};

template <typename T>
__global__ void __launch_bounds__(kPrologueWarps * 32)
fipa_prologue_kernel(const PrologueArgs a) {
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

  const int t = blockIdx.x, b = blockIdx.y;
  const int N = p.N, H = p.H, P = p.P, Q = p.Q, RCz = p.R * p.Cz;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  extern __shared__ float sh[];
  __shared__ float red[kPrologueWarps][4];
  __shared__ float4 s_orig;

  // ---- tile origin: mean translation of the valid residues of the tile
  {
    float sx = 0.f, sy = 0.f, sz = 0.f, cnt = 0.f;
    if (threadIdx.x < kTile) {
      const int i = t * kTile + threadIdx.x;
      if (i < N && a.in.mask[(size_t)b * N + i]) {
        const size_t o = ((size_t)b * N + i) * 3;
        sx = ld_in(tr, o + 0); sy = ld_in(tr, o + 1); sz = ld_in(tr, o + 2); cnt = 1.f;
      }
    }
    for (int off = 16; off; off >>= 1) {
      sx += __shfl_xor_sync(0xffffffffu, sx, off);
      sy += __shfl_xor_sync(0xffffffffu, sy, off);
      sz += __shfl_xor_sync(0xffffffffu, sz, off);
      cnt += __shfl_xor_sync(0xffffffffu, cnt, off);
    }
    if (lane == 0) { red[warp][0] = sx; red[warp][1] = sy; red[warp][2] = sz; red[warp][3] = cnt; }
    __syncthreads();
    if (threadIdx.x == 0) {
      float ax = 0.f, ay = 0.f, az = 0.f, ac = 0.f;
      for (int wi = 0; wi < kTile / 32; ++wi) { ax += red[wi][0]; ay += red[wi][1]; az += red[wi][2]; ac += red[wi][3]; }
      const float inv = ac > 0.f ? 1.f / ac : 0.f;
      s_orig = make_float4(ax * inv, ay * inv, az * inv, ac);
      a.w.orig[(size_t)b * p.nT + t] = s_orig;
      a.w.flag[(size_t)b * p.nT + t] = ac > 0.f ? 1 : 0;
    }
    __syncthreads();
  }
  const float ox = s_orig.x, oy = s_orig.y, oz = s_orig.z;

  // per-warp scratch: a' [P*3], b' [P*3], g' [Q*3], z1 row [R*Cz]
  const int PQ = P > Q ? P : Q;
  float* pa = sh + (size_t)warp * (9 * PQ + RCz);
  float* pb = pa + 3 * PQ;
  float* pg = pb + 3 * PQ;
  float* z1s = pg + 3 * PQ;
  const float sqk = rsqrtf(3.0f * (float)p.D);
  const float inv_sqrt3 = rsqrtf(3.0f);

  for (int r = warp; r < kTile; r += kPrologueWarps) {
    const int i = t * kTile + r;
    if (i >= N) break;
    const size_t bi = (size_t)b * N + i;
    const bool valid = a.in.mask[bi] != 0;
    float R[9], tv[3];
#pragma unroll
    for (int e = 0; e < 9; ++e) R[e] = ld_in(rot, bi * 9 + e);
#pragma unroll
    for (int e = 0; e < 3; ++e) tv[e] = ld_in(tr, bi * 3 + e);
    const float tx = tv[0] - ox, ty = tv[1] - oy, tz = tv[2] - oz;   // t_i - o_T

    // pair factors of this residue: z2 row goes to Z, z1 row to scratch
    __half* zrow = a.w.Z + bi * p.Zp;
    for (int e = lane; e < RCz; e += 32) {
      z1s[e] = ld_in(z1, bi * RCz + e);
      const float x = valid ? ld_in(z2, bi * RCz + e) : 0.f;
      for (int seg = 0; seg < p.nz; ++seg) zrow[seg * RCz + e] = part(x, seg == 1);
    }
    for (int c = p.Zc + lane; c < p.Zp; c += 32) zrow[c] = __float2half_rn(0.f);
    __syncwarp();

    for (int h = 0; h < H; ++h) {
      const float g = point_weight(ld_in(raw, h), P);
      const size_t bhi = ((size_t)b * H + h) * N + i;
      const size_t in_pts = (bi * H + h);
      // global points relative to the tile origin
      for (int e = lane; e < PQ; e += 32) {
        if (e < P) {
          float x0 = ld_in(qp, (in_pts * P + e) * 3 + 0), x1 = ld_in(qp, (in_pts * P + e) * 3 + 1),
                x2 = ld_in(qp, (in_pts * P + e) * 3 + 2);
          pa[e * 3 + 0] = R[0] * x0 + R[1] * x1 + R[2] * x2 + tx;
          pa[e * 3 + 1] = R[3] * x0 + R[4] * x1 + R[5] * x2 + ty;
          pa[e * 3 + 2] = R[6] * x0 + R[7] * x1 + R[8] * x2 + tz;
          x0 = ld_in(kp, (in_pts * P + e) * 3 + 0); x1 = ld_in(kp, (in_pts * P + e) * 3 + 1);
          x2 = ld_in(kp, (in_pts * P + e) * 3 + 2);
          pb[e * 3 + 0] = R[0] * x0 + R[1] * x1 + R[2] * x2 + tx;
          pb[e * 3 + 1] = R[3] * x0 + R[4] * x1 + R[5] * x2 + ty;
          pb[e * 3 + 2] = R[6] * x0 + R[7] * x1 + R[8] * x2 + tz;
        }
        if (e < Q) {
          const float x0 = ld_in(vp, (in_pts * Q + e) * 3 + 0), x1 = ld_in(vp, (in_pts * Q + e) * 3 + 1),
                      x2 = ld_in(vp, (in_pts * Q + e) * 3 + 2);
          pg[e * 3 + 0] = R[0] * x0 + R[1] * x1 + R[2] * x2 + tx;
          pg[e * 3 + 1] = R[3] * x0 + R[4] * x1 + R[5] * x2 + ty;
          pg[e * 3 + 2] = R[6] * x0 + R[7] * x1 + R[8] * x2 + tz;
        }
      }
      __syncwarp();

      // ---- lifted query row
      __half* qrow = a.w.Q + bhi * p.Kq;
      const float vs = valid ? 1.f : 0.f;
      for (int seg = 0; seg < p.nsq; ++seg)
        for (int d = lane; d < p.D; d += 32)
          qrow[seg * p.D + d] = part(vs * ld_in(q, in_pts * p.D + d) * sqk, seg == 2);
      {
        const int base = p.nsq * p.D, n3 = 3 * P;
        for (int seg = 0; seg < 3; ++seg)
          for (int e = lane; e < n3; e += 32) qrow[base + seg * n3 + e] = part(vs * 2.f * g * pa[e], seg == 2);
        for (int c = p.KHc + lane; c < p.KHp; c += 32) qrow[c] = __float2half_rn(0.f);
      }
      for (int seg = 0; seg < p.nz; ++seg)
        for (int rr = 0; rr < p.R; ++rr)
          for (int c = lane; c < p.Cz; c += 32) {
            const float u = vs * z1s[rr * p.Cz + c] * ld_in(Wb, (size_t)c * H + h) * inv_sqrt3;
            qrow[p.KHp + seg * RCz + rr * p.Cz + c] = part(u, seg == 2);
          }
      for (int c = p.KHp + p.Zc + lane; c < p.Kq; c += 32) qrow[c] = __float2half_rn(0.f);

      // ---- lifted key row (head part)
      __half* krow = a.w.KH + bhi * p.KHp;
      for (int seg = 0; seg < p.nsq; ++seg)
        for (int d = lane; d < p.D; d += 32) krow[seg * p.D + d] = part(vs * ld_in(k, in_pts * p.D + d), seg == 1);
      {
        const int base = p.nsq * p.D, n3 = 3 * P;
        for (int seg = 0; seg < 3; ++seg)
          for (int e = lane; e < n3; e += 32) krow[base + seg * n3 + e] = part(vs * pb[e], seg == 1);
        for (int c = p.KHc + lane; c < p.KHp; c += 32) krow[c] = __float2half_rn(0.f);
      }

      // ---- lifted value row (head part)
      __half* vrow = a.w.VH + bhi * p.VHp;
      for (int seg = 0; seg < p.nsv; ++seg)
        for (int d = lane; d < p.Dv; d += 32) vrow[seg * p.Dv + d] = part(vs * ld_in(v, in_pts * p.Dv + d), seg == 1);
      {
        const int base = p.nsv * p.Dv, n3 = 3 * Q;
        for (int seg = 0; seg < 2; ++seg)
          for (int e = lane; e < n3; e += 32) vrow[base + seg * n3 + e] = part(vs * pg[e], seg == 1);
        for (int c = p.VHc + lane; c < p.VHp; c += 32) vrow[c] = __float2half_rn(0.f);
      }

      // ---- per-key and per-query fp32 corrections
      if (lane == 0) {
        float Ax = 0.f, Ay = 0.f, Az = 0.f, a2 = 0.f, Bx = 0.f, By = 0.f, Bz = 0.f, b2 = 0.f;
        for (int e = 0; e < P; ++e) {
          Ax += pa[3 * e]; Ay += pa[3 * e + 1]; Az += pa[3 * e + 2];
          a2 += pa[3 * e] * pa[3 * e] + pa[3 * e + 1] * pa[3 * e + 1] + pa[3 * e + 2] * pa[3 * e + 2];
          Bx += pb[3 * e]; By += pb[3 * e + 1]; Bz += pb[3 * e + 2];
          b2 += pb[3 * e] * pb[3 * e] + pb[3 * e + 1] * pb[3 * e + 1] + pb[3 * e + 2] * pb[3 * e + 2];
        }
        a.w.kvec[bhi] = valid ? make_float4(-g * b2, Bx, By, Bz) : make_float4(-INFINITY, 0.f, 0.f, 0.f);
        a.w.qvec[bhi] = make_float4(Ax, Ay, Az, -g * a2);
      }
      __syncwarp();
    }
  }
}

}  // namespace

cudaError_t launch_prologue(const Plan& p, const Inputs& in, const Work& w, cudaStream_t s) {
  PrologueArgs a{p, in, w};
  const int PQ = p.P > p.Q ? p.P : p.Q;
  const size_t smem = (size_t)kPrologueWarps * (9 * PQ + p.R * p.Cz) * sizeof(float);
  dim3 grid(p.nT, p.B);
  if (p.f32) {
    auto kfn = fipa_prologue_kernel<float>;
    cudaError_t e = cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kfn<<<grid, kPrologueWarps * 32, smem, s>>>(a);
  } else {
    auto kfn = fipa_prologue_kernel<__nv_bfloat16>;
    cudaError_t e = cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kfn<<<grid, kPrologueWarps * 32, smem, s>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace fipa
