// prologue.cu -- frames to global points and the lifted Q / K / V rows (HBM-bound).
//
// One launch: CTAs that prepare the output weights (wprep.cuh), then one lift
// CTA per 8 residues of a sample, all heads.  A lift CTA reduces the origin o_G
// of its 32-residue group (mean translation of its valid residues) and the
// valid flag of its 128-residue tile; it stages the frames, z1 rows and Wb^T in
// shared memory, applies every frame T_i(x) = R_i x + t_i (page "Invariant
// point attention (IPA)", Required behavior: column-vector convention) to all
// query / key / value points in parallel, and then writes every lifted row of
// plan.h as 16-byte chunks of 8 fp16 values.  Each column segment is padded to
// a multiple of 8, so a chunk never straddles two segments.
// The distance weight g is folded into the query point columns, following the
// squared-norm expansion of FlashIPA's lifted attention.
#include "kernels.h"
#include "sm100.cuh"
#include "wprep.cuh"

namespace fipa {
namespace {

constexpr int kLiftThreads = 256;

struct PrologueArgs {
  Plan p;
  Inputs in;
  Work w;
};

// ---- lift: chunk descriptors
// Every 16-byte chunk (8 fp16 columns) of a lifted row reads 8 consecutive
// fp32 values of one zero-padded source row in shared memory.  A per-CTA table
// holds, for each chunk position of each row type, which source it reads, at
// which offset, and whether it stores the hi or the lo half; the write loop
// then does no index arithmetic beyond one table load per chunk.
enum : uint32_t { kSrcZero = 0, kSrcScalar = 1, kSrcPoint = 2, kSrcPair = 3, kSrcZ2 = 4, kSrcOne = 5 };
enum : int { kRowQ = 0, kRowK = 1, kRowV = 2, kRowZ = 3 };

__device__ __forceinline__ uint32_t make_desc(uint32_t src, int off, int woff, bool lo) {
  return (uint32_t)off | ((uint32_t)woff << 11) | (src << 22) | ((lo ? 1u : 0u) << 26);
}

// Descriptor of the chunk starting at column `col` of a row of type `rt`,
// following the column layout of plan.h.  Point offsets index the per-(residue,
// head) point row [a' (P38) | b' (P38) | g' (Q38)].
__device__ uint32_t chunk_desc(const Plan& p, int rt, int col) {
  const int RCz = p.R * p.Cz;
  if (rt == kRowZ) {
    const int seg = col / p.RC8, e0 = col - seg * p.RC8;
    return seg < p.nz ? make_desc(kSrcZ2, e0, 0, seg == 1) : make_desc(kSrcZero, 0, 0, false);
  }
  if (rt == kRowV) {
    const int sv = p.nsv * p.Dv8;
    if (col < sv) {
      const int seg = col / p.Dv8;
      return make_desc(kSrcScalar, col - seg * p.Dv8, 0, seg == 1);
    }
    if (col < sv + 2 * p.Q38) {
      const int seg = (col - sv) / p.Q38;
      return make_desc(kSrcPoint, 2 * p.P38 + (col - sv - seg * p.Q38), 0, seg == 1);
    }
    // float32 inputs: a column of ones (its own chunk; VHc is a multiple of 8)
    if (col == p.ones_col) return make_desc(kSrcOne, 0, 0, false);
    return make_desc(kSrcZero, 0, 0, false);
  }
  // query (rt 0) and key (rt 1) head parts: the lo copy is segment 2 on the
  // query side and segment 1 on the key side
  const int lo_seg = rt == kRowQ ? 2 : 1;
  const int sq = p.nsq * p.D8;
  if (col < sq) {
    const int seg = col / p.D8;
    return make_desc(kSrcScalar, col - seg * p.D8, 0, seg == lo_seg);
  }
  if (col < p.KHp) {
    if (!p.geo_simt && col < sq + 3 * p.P38) {
      const int seg = (col - sq) / p.P38;
      return make_desc(kSrcPoint, (rt == kRowQ ? 0 : p.P38) + (col - sq - seg * p.P38), 0, seg == lo_seg);
    }
    return make_desc(kSrcZero, 0, 0, false);
  }
  // query pair part: u = z1[r,c] Wb[c,h] / sqrt(3)
  const int cc = col - p.KHp;
  int e0;
  bool lo;
  if (p.nqz == 2) {                       // [u hi | u lo], each Zp wide
    lo = cc >= p.Zp;
    e0 = lo ? cc - p.Zp : cc;
  } else {                                // [u hi | u hi | u lo], RC8 apart
    const int seg = cc / p.RC8;
    e0 = seg < p.nz ? cc - seg * p.RC8 : RCz;
    lo = (seg == 2);
  }
  if (e0 >= RCz) return make_desc(kSrcZero, 0, 0, false);
  const int rr = e0 / p.Cz;
  return make_desc(kSrcPair, e0, e0 - rr * p.Cz, lo);
}

__device__ __forceinline__ void lds8(const float* src, float (&v)[8]) {
  const float4 a = reinterpret_cast<const float4*>(src)[0], b = reinterpret_cast<const float4*>(src)[1];
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
__device__ __forceinline__ void sts8(float* dst, const float (&v)[8]) {
  reinterpret_cast<float4*>(dst)[0] = make_float4(v[0], v[1], v[2], v[3]);
  reinterpret_cast<float4*>(dst)[1] = make_float4(v[4], v[5], v[6], v[7]);
}
__device__ __forceinline__ uint32_t h2_bits(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }
// Round 8 values to fp16 (hi), or store the rounding residual x - fp16(x) (lo).
__device__ __forceinline__ void stg8_half(__half* dst, const float (&v)[8], bool lo) {
  uint32_t w[4];
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    const __half2 h = __floats2half2_rn(v[2 * t], v[2 * t + 1]);
    if (lo) {
      const float2 f = __half22float2(h);
      w[t] = h2_bits(__floats2half2_rn(v[2 * t] - f.x, v[2 * t + 1] - f.y));
    } else {
      w[t] = h2_bits(h);
    }
  }
  *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
}

// 8 consecutive inputs as fp32 (16-byte aligned source: one or two vector loads).
__device__ __forceinline__ void ldg8(const float* src, float (&v)[8]) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(src)), b = __ldg(reinterpret_cast<const float4*>(src) + 1);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
__device__ __forceinline__ void ldg8(const __nv_bfloat16* src, float (&v)[8]) {
  const uint4 u = __ldg(reinterpret_cast<const uint4*>(src));
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    v[2 * t] = __uint_as_float(w[t] << 16);
    v[2 * t + 1] = __uint_as_float(w[t] & 0xffff0000u);
  }
}

// Stage `nrows` contiguous input rows of L values into shared rows of L8
// (a multiple of 8; fd_vec divides by L8 / 8) floats, times `scale`, zero-padded.
template <typename T>
__device__ __forceinline__ void stage_rows(float* dst, int L8, const FastDiv& fd_vec, const T* src, int L,
                                           int nrows, float scale) {
  const uint32_t nvec = L8 >> 3;
  const bool vec = (L & 7) == 0 && (reinterpret_cast<uintptr_t>(src) & 15) == 0;
  for (uint32_t e = threadIdx.x; e < (uint32_t)nrows * nvec; e += blockDim.x) {
    const uint32_t r = fd_vec.div(e), c = (e - r * nvec) << 3;
    float v[8];
    if (vec) {
      ldg8(src + (size_t)r * L + c, v);
    } else {
#pragma unroll
      for (int t = 0; t < 8; ++t) v[t] = (int)c + t < L ? ld_in(src, (size_t)r * L + c + t) : 0.f;
    }
#pragma unroll
    for (int t = 0; t < 8; ++t) v[t] *= scale;
    sts8(dst + (size_t)r * L8 + c, v);
  }
}

// The 8 fp32 values of one chunk of a lifted row (all zero for a masked residue).
__device__ __forceinline__ void chunk_values(uint32_t d, bool valid, const float* scal, const float* prow,
                                             float ptscale, const float* z1row, const float* wrow, int Cz, bool cz8,
                                             float (&v)[8]) {
  const uint32_t src = valid ? (d >> 22) & 15u : (uint32_t)kSrcZero;
  const int off = d & 2047, woff = (d >> 11) & 2047;
  if (src == kSrcScalar) {
    lds8(scal + off, v);
  } else if (src == kSrcPoint) {
    lds8(prow + off, v);
#pragma unroll
    for (int t = 0; t < 8; ++t) v[t] = ptscale * v[t];
  } else if (src == kSrcOne) {
#pragma unroll
    for (int t = 0; t < 8; ++t) v[t] = t == 0 ? 1.f : 0.f;
  } else if (src == kSrcPair) {
    float w[8];
    lds8(z1row + off, v);
    if (cz8) {
      lds8(wrow + woff, w);
    } else {
      int cw = woff;
#pragma unroll
      for (int t = 0; t < 8; ++t) { w[t] = wrow[cw]; if (++cw == Cz) cw = 0; }
    }
#pragma unroll
    for (int t = 0; t < 8; ++t) v[t] *= w[t];
  } else {
#pragma unroll
    for (int t = 0; t < 8; ++t) v[t] = 0.f;
  }
}

template <typename T>
__global__ void __launch_bounds__(kLiftThreads) fipa_lift_kernel(const PrologueArgs a) {
  const Plan& p = a.p;
  const T* qp = static_cast<const T*>(a.in.q_pts);
  const T* kp = static_cast<const T*>(a.in.k_pts);
  const T* vp = static_cast<const T*>(a.in.v_pts);
  const T* rot = static_cast<const T*>(a.in.rot);
  const T* tr = static_cast<const T*>(a.in.trans);
  const T* Wb = static_cast<const T*>(a.in.Wb);
  const T* raw = static_cast<const T*>(a.in.raw);
  const int N = p.N, H = p.H, P = p.P, Q = p.Q, Cz = p.Cz, RCz = p.R * p.Cz;
  extern __shared__ float4 sh4[];
  if ((int)blockIdx.x < p.wp_ctas) {
    // output-weight preparation (independent of the lift)
    const int nbx = cdiv(p.F, 32), cout_pad = rup(p.Cout, p.ntile_out);
    const int ntiles = nbx * cdiv(cout_pad, 32);
    for (int t = blockIdx.x * kWpTiles; t < min(ntiles, (int)(blockIdx.x + 1) * kWpTiles); ++t) {
      const int by = t / nbx, bx = t - by * nbx;
      weight_prep_tile(p, static_cast<const T*>(a.in.w_out), a.w.wT, cout_pad, bx, by,
                       reinterpret_cast<float (*)[33]>(sh4));
      __syncthreads();                      // the tile buffer is reused by the next tile
    }
    return;
  }
  const int lid = blockIdx.x - p.wp_ctas;
  const int LR = p.lift_res;                 // residues per CTA (4 or 8; all in one 32-residue group)
  const int b = lid / p.lift_ctas, i0 = (lid - b * p.lift_ctas) * LR;
  const int nres = min(LR, N - i0);
  const int RH = nres * H;
  const int PW = 2 * p.P38 + p.Q38;            // point row: [a' | b' | g'], each segment zero-padded
  const int nQ8 = p.Kq >> 3, nK8 = p.KHp >> 3, nV8 = p.VHp >> 3, nZ8 = p.Zp >> 3;

  float* wbt = reinterpret_cast<float*>(sh4);                // [H][Cz]  Wb^T / sqrt(3)
  float* z1s = wbt + rup(H * Cz, 8);                         // [LR][RC8]
  float* qs = z1s + LR * p.RC8;                              // [LR*H][D8]  q / sqrt(3D)
  float* ks = qs + LR * H * p.D8;                            // [LR*H][D8]
  float* vs = ks + LR * H * p.D8;                            // [LR*H][Dv8]
  float* pts = vs + LR * H * p.Dv8;                          // [LR*H][PW]  global point - o_G
  float* frm = pts + LR * H * PW;                            // [LR][12]  R (row-major), t
  uint32_t* tab = reinterpret_cast<uint32_t*>(frm + LR * 12);   // chunk descriptors Q | K | V | Z
  __shared__ float s_gamma[64];
  __shared__ int s_valid[kLiftRes];
  __shared__ float4 s_orig;

  // ---- phase 0: origin o_G of this CTA's 32-residue group (mean translation
  // of its valid residues; its CTA at the group start writes it for the core),
  // and the valid flag of the 128-residue tile (written by its first CTA)
  const int warp0 = threadIdx.x >> 5, lane0 = threadIdx.x & 31;
  if (warp0 == 0) {
    const int g = i0 / kGroup, i = g * kGroup + lane0;
    float sx = 0.f, sy = 0.f, sz = 0.f, cnt = 0.f;
    if (i < N && a.in.mask[(size_t)b * N + i]) {
      const size_t o = ((size_t)b * N + i) * 3;
      sx = ld_in(tr, o + 0); sy = ld_in(tr, o + 1); sz = ld_in(tr, o + 2); cnt = 1.f;
    }
    for (int off = 16; off; off >>= 1) {
      sx += __shfl_xor_sync(0xffffffffu, sx, off);
      sy += __shfl_xor_sync(0xffffffffu, sy, off);
      sz += __shfl_xor_sync(0xffffffffu, sz, off);
      cnt += __shfl_xor_sync(0xffffffffu, cnt, off);
    }
    if (lane0 == 0) {
      const float inv = cnt > 0.f ? 1.f / cnt : 0.f;
      s_orig = make_float4(sx * inv, sy * inv, sz * inv, cnt);
      if (i0 % kGroup == 0) a.w.orig[(size_t)b * p.nG + g] = s_orig;
    }
  } else if (warp0 == 1 && i0 % kTile == 0) {
    bool any = false;
    for (int k = lane0; k < kTile; k += 32) {
      const int i = i0 + k;
      any |= i < N && a.in.mask[(size_t)b * N + i] != 0;
    }
    any = __any_sync(0xffffffffu, any);
    if (lane0 == 0) a.w.flag[(size_t)b * p.nT + i0 / kTile] = any ? 1 : 0;
    // groups of this tile that lie wholly past N have no lift CTA: their
    // origin is 0 with no valid residue (every tile's four are read by the core)
    if (lane0 < kTile / kGroup && i0 + lane0 * kGroup >= N)
      a.w.orig[(size_t)b * p.nG + i0 / kGroup + lane0] = make_float4(0.f, 0.f, 0.f, 0.f);
  }

  // ---- phase 1 (with phase 0 above): stage the inputs of the 8 residues,
  // zero the point rows, build the chunk table (independent work, issued
  // together)
  const float inv_sqrt3 = rsqrtf(3.0f);
  const size_t bi0 = (size_t)b * N + i0;
  for (uint32_t e = threadIdx.x; e < (uint32_t)(H * Cz); e += blockDim.x) {
    const uint32_t h = p.fd_Cz.div(e), c = e - h * Cz;
    wbt[e] = ld_in(Wb, (size_t)c * H + h) * inv_sqrt3;
  }
  stage_rows(z1s, p.RC8, p.fd_RC8v, static_cast<const T*>(a.in.z1) + bi0 * RCz, RCz, nres, 1.f);
  stage_rows(qs, p.D8, p.fd_D8v, static_cast<const T*>(a.in.q) + bi0 * H * p.D, p.D, RH,
             rsqrtf(3.0f * (float)p.D));
  stage_rows(ks, p.D8, p.fd_D8v, static_cast<const T*>(a.in.k) + bi0 * H * p.D, p.D, RH, 1.f);
  stage_rows(vs, p.Dv8, p.fd_Dv8v, static_cast<const T*>(a.in.v) + bi0 * H * p.Dv, p.Dv, RH, 1.f);
  for (int e = threadIdx.x; e < (RH * PW) >> 2; e += blockDim.x)
    reinterpret_cast<float4*>(pts)[e] = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int e = threadIdx.x; e < nres * 12; e += blockDim.x) {
    const int r = e / 12, c = e - r * 12;
    const size_t bi = bi0 + r;
    frm[e] = c < 9 ? ld_in(rot, bi * 9 + c) : ld_in(tr, bi * 3 + (c - 9));   // t - o_G in phase 2
  }
  for (int c = threadIdx.x; c < nQ8 + nK8 + nV8 + nZ8; c += blockDim.x) {
    int rt = kRowQ, cc = c;
    if (cc >= nQ8) { cc -= nQ8; rt = kRowK;
      if (cc >= nK8) { cc -= nK8; rt = kRowV;
        if (cc >= nV8) { cc -= nV8; rt = kRowZ; } } }
    tab[c] = chunk_desc(p, rt, cc << 3);
  }
  for (int h = threadIdx.x; h < H && h < 64; h += blockDim.x) s_gamma[h] = point_weight(ld_in(raw, h), P);
  if (threadIdx.x < nres) s_valid[threadIdx.x] = a.in.mask[bi0 + threadIdx.x] != 0;
  __syncthreads();

  // ---- phase 2: every point of every head, T_i(x) = R_i x + t_i relative to
  // the group origin (page "Invariant point attention (IPA)", Required
  // behavior: column-vector convention)
  const float4 og = s_orig;                    // all of the CTA's residues share one group
  auto apply = [&](const T* src, int npts, const FastDiv& fd_npts, int seg_off) {
    for (uint32_t e = threadIdx.x; e < (uint32_t)(RH * npts); e += blockDim.x) {
      const uint32_t rh = fd_npts.div(e), pt = e - rh * npts, r = p.fd_H.div(rh);
      const T* x = src + ((bi0 * H + rh) * npts + pt) * 3;
      const float x0 = ld_in(x, 0), x1 = ld_in(x, 1), x2 = ld_in(x, 2);
      const float* F = frm + r * 12;
      const float t0 = F[9] - og.x, t1 = F[10] - og.y, t2 = F[11] - og.z;
      float* o = pts + (size_t)rh * PW + seg_off + 3 * pt;
      o[0] = F[0] * x0 + F[1] * x1 + F[2] * x2 + t0;
      o[1] = F[3] * x0 + F[4] * x1 + F[5] * x2 + t1;
      o[2] = F[6] * x0 + F[7] * x1 + F[8] * x2 + t2;
    }
  };
  apply(qp, P, p.fd_P, 0);
  apply(kp, P, p.fd_P, p.P38);
  apply(vp, Q, p.fd_Q, 2 * p.P38);
  __syncthreads();

  // ---- phase 3a: per (residue, head) fp32 corrections (and the fp32 points
  // of float32 mode)
  for (uint32_t e = threadIdx.x; e < (uint32_t)RH; e += blockDim.x) {
    const uint32_t r = p.fd_H.div(e), h = e - r * H;
    const float g = s_gamma[h < 64 ? h : 63];
    const float* pa = pts + (size_t)e * PW;
    const float* pb = pa + p.P38;
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

  // ---- phase 3b: every lifted row, one pass per row type over all (row,
  // chunk) pairs of the CTA: consecutive threads write consecutive 16-byte
  // chunks of a row
  const bool cz8 = (Cz & 7) == 0;
  const uint32_t nthr = blockDim.x;
  // with the [u hi | u lo] pair layout a u-hi chunk also writes its lo
  // partner (the same products, the rounding residual instead of the value)
  const uint32_t uhi0 = (uint32_t)p.KHp >> 3, zch = (uint32_t)p.Zp >> 3;
  const bool pair_lo = p.nqz == 2;
  // bfloat16 inputs with Cz a multiple of 8: the u chunks [u hi | u lo] of the
  // Qhat rows get a loop of their own (no chunk table, no source dispatch);
  // the table loop below then covers the head part only
  const bool upath = !p.f32 && cz8;
  if (upath) {
    const uint32_t RCz8 = (uint32_t)RCz >> 3;
    for (uint32_t e = threadIdx.x; e < (uint32_t)RH * zch; e += nthr) {
      const uint32_t rh = p.fd_nZ8.div(e), j = e - rh * zch, r = p.fd_H.div(rh), h = rh - r * H;
      float v[8];
      if (j < RCz8 && s_valid[r] != 0) {
        const uint32_t col = j << 3, cw = col - p.fd_Cz.div(col) * (uint32_t)Cz;   // channel c of column (r', c)
        float w[8];
        lds8(z1s + (size_t)r * p.RC8 + col, v);
        lds8(wbt + (size_t)h * Cz + cw, w);
#pragma unroll
        for (int t = 0; t < 8; ++t) v[t] *= w[t];
      } else {
#pragma unroll
        for (int t = 0; t < 8; ++t) v[t] = 0.f;
      }
      __half* urow = a.w.Q + (((size_t)b * H + h) * N + i0 + r) * p.Kq + p.KHp + ((size_t)j << 3);
      stg8_half(urow, v, false);
      if (pair_lo) stg8_half(urow + p.Zp, v, true);
    }
  }
  const FastDiv& fdq = upath ? p.fd_nK8 : p.fd_nQ8e;
  const uint32_t nQ8e = fdq.d;
  for (uint32_t e = threadIdx.x; e < (uint32_t)RH * nQ8e; e += nthr) {
    const uint32_t rh = fdq.div(e), c = e - rh * nQ8e, r = p.fd_H.div(rh), h = rh - r * H;
    const uint32_t d = tab[c];
    float v[8];
    chunk_values(d, s_valid[r] != 0, qs + (size_t)rh * p.D8, pts + (size_t)rh * PW, 2.f * s_gamma[h < 64 ? h : 63],
                 z1s + (size_t)r * p.RC8, wbt + (size_t)h * Cz, Cz, cz8, v);
    __half* qrow = a.w.Q + (((size_t)b * H + h) * N + i0 + r) * p.Kq;
    stg8_half(qrow + ((size_t)c << 3), v, (d >> 26) & 1u);
    if (pair_lo && c >= uhi0) stg8_half(qrow + ((size_t)(c + zch) << 3), v, true);
  }
  for (uint32_t e = threadIdx.x; e < (uint32_t)RH * nK8; e += nthr) {
    const uint32_t rh = p.fd_nK8.div(e), c = e - rh * nK8, r = p.fd_H.div(rh), h = rh - r * H;
    const uint32_t d = tab[nQ8 + c];
    float v[8];
    chunk_values(d, s_valid[r] != 0, ks + (size_t)rh * p.D8, pts + (size_t)rh * PW, 1.f, nullptr, nullptr, Cz,
                 cz8, v);
    stg8_half(a.w.KH + (((size_t)b * H + h) * N + i0 + r) * p.KHp + ((size_t)c << 3), v, (d >> 26) & 1u);
  }
  for (uint32_t e = threadIdx.x; e < (uint32_t)RH * nV8; e += nthr) {
    const uint32_t rh = p.fd_nV8.div(e), c = e - rh * nV8, r = p.fd_H.div(rh), h = rh - r * H;
    const uint32_t d = tab[nQ8 + nK8 + c];
    float v[8];
    chunk_values(d, s_valid[r] != 0, vs + (size_t)rh * p.Dv8, pts + (size_t)rh * PW, 1.f, nullptr, nullptr, Cz,
                 cz8, v);
    stg8_half(a.w.VH + (((size_t)b * H + h) * N + i0 + r) * p.VHp + ((size_t)c << 3), v, (d >> 26) & 1u);
  }
  // pair-factor rows read z2 straight from global memory (one use per value)
  const T* z2 = static_cast<const T*>(a.in.z2);
  const bool z2vec = (RCz & 7) == 0 && (reinterpret_cast<uintptr_t>(z2) & 15) == 0;
  for (uint32_t e = threadIdx.x; e < (uint32_t)nres * nZ8; e += nthr) {
    const uint32_t r = p.fd_nZ8.div(e), c = e - r * nZ8;
    const uint32_t d = tab[nQ8 + nK8 + nV8 + c];
    float v[8];
    const int off = d & 2047;
    if (s_valid[r] != 0 && ((d >> 22) & 15u) == kSrcZ2) {
      const T* zr = z2 + (bi0 + r) * RCz + off;
      if (z2vec && off + 8 <= RCz) {
        ldg8(zr, v);
      } else {
#pragma unroll
        for (int t = 0; t < 8; ++t) v[t] = off + t < RCz ? ld_in(zr, t) : 0.f;
      }
    } else {
#pragma unroll
      for (int t = 0; t < 8; ++t) v[t] = 0.f;
    }
    stg8_half(a.w.Z + (bi0 + r) * p.Zp + ((size_t)c << 3), v, (d >> 26) & 1u);
  }
}

}  // namespace

cudaError_t launch_prologue(const Plan& p, const Inputs& in, const Work& w, cudaStream_t s) {
  // one launch: the weight-preparation CTAs first, then B x lift_ctas lift CTAs
  PrologueArgs a{p, in, w};
  const unsigned grid = (unsigned)(p.wp_ctas + (size_t)p.B * p.lift_ctas);
  const void* kfn = p.in_f32 ? reinterpret_cast<const void*>(fipa_lift_kernel<float>)
                             : reinterpret_cast<const void*>(fipa_lift_kernel<__nv_bfloat16>);
  cudaError_t e = allow_max_smem(kfn);
  if (e != cudaSuccess) return e;
  if (p.in_f32)
    fipa_lift_kernel<float><<<grid, kLiftThreads, p.lift_smem, s>>>(a);
  else
    fipa_lift_kernel<__nv_bfloat16><<<grid, kLiftThreads, p.lift_smem, s>>>(a);
  return cudaGetLastError();
}

}  // namespace fipa
