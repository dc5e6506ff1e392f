// plan.h -- derived sizes and device-workspace layout of one fused IPA forward.
//
// Lifted operand layout (FlashIPA, "Flash Invariant Point Attention": the
// squared-norm expansion |a-b|^2 = |a|^2 - 2 a.b + |b|^2 turns the point
// term into a dot product; the pair factors z1, z2 turn the pair bias and the
// pair aggregation into dot products).  Rows are fp16; a 16-bit value that
// needs more precision is stored as hi + lo halves and the partner operand
// repeats its own hi half, so hi*hi + hi*lo + lo*hi restores ~22 bits.
//
//   Qhat [B*H, N, Kq]  = [ QH (KHp cols) | QZ (Zp cols) ]
//       QH   bf16 mode: [ q/sqrt(3D) | 2g a' hi | 2g a' hi | 2g a' lo | 0.. ]
//            f32  mode: [ q/sqrt(3D) hi | hi | lo | 2g a' hi | hi | lo | 0.. ]
//       QZ   bf16 mode: [ z1[r,c] Wb[c,h] / sqrt(3) ]          (r-major, then c)
//            f32  mode: [ u hi | u hi | u lo ]
//   KH   [B*H, N, KHp]  bf16: [ k | b' hi | b' lo | b' hi | 0.. ]
//                        f32: [ k hi | lo | hi | b' hi | lo | hi | 0.. ]
//   Z    [B,   N, Zp ]  bf16: [ z2 ]            f32: [ z2 hi | z2 lo | z2 hi ]
//   VH   [B*H, N, VHp]  bf16: [ v | g' hi | g' lo | 0.. ]
//                        f32: [ v hi | v lo | g' hi | g' lo | 0.. ]
// where a' = T_i(q_p) - o_T, b' = T_j(k_p) - o_T, g' = T_j(v_q) - o_T are
// global points relative to the mean translation o_T of their own 128-residue
// tile, and g = the per-head distance weight.  The value side uses the first
// ZV columns of Z (f32 mode: z2 hi | z2 lo).
#pragma once

#include <stddef.h>
#include <stdint.h>

namespace fipa {

constexpr int kTile = 128;       // residues per query / key tile (MMA M and N)
constexpr int kChunk = 64;       // fp16 columns per 128-byte swizzled chunk
constexpr int kTmemS = 0;        // TMEM column of the logit tile S (128 fp32 columns)
constexpr int kTmemP = 128;      // TMEM column of P (fp16 pairs: 64 columns, 128 when split)
constexpr int kMaxQChunks = 8;   // resident Qhat tile <= 128 KB of shared memory
constexpr int kMaxPts = 64;      // points per head handled by the prologue scratch
constexpr int kMaxRCz = 1024;    // R*Cz handled by the prologue scratch
constexpr int kMaxTiles = 2048;  // key tiles per sample (N <= 262144)

static inline int cdiv(int a, int b) { return (a + b - 1) / b; }
static inline int rup(int a, int b) { return cdiv(a, b) * b; }
static inline size_t rup_sz(size_t a, size_t b) { return (a + b - 1) / b * b; }

struct Plan {
  int B, N, H, D, Dv, P, Q, Cz, R, Cout, F;
  int f32;            // 1: float32 inputs (hi/lo splits everywhere); 0: bfloat16 inputs
  int nT;             // tiles per sample
  int nsq;            // copies of the scalar q/k columns (1 or 3)
  int nsv;            // copies of the scalar v columns (1 or 2)
  int nz;             // copies of the pair columns on the key side (1 or 3)
  int nzv;            // copies of the pair columns on the value side (1 or 2)
  int KHc, KHp, nKH;  // key/query head-part columns, padded, chunks
  int Zc, Zp, nZ;     // pair columns, padded, chunks
  int Kq, nQc;        // Qhat row width and chunks
  int VHc, VHp, nVH;  // value head-part columns, padded, chunks
  int ZVc, nZV;       // pair columns used by the value product, chunks
  int Ocols;          // VHp + nZV * 64: fp32 accumulator columns per row
  int Pcols;          // TMEM columns holding P (64, or 128 for hi+lo)
  int tmemO;          // TMEM column of the O accumulator
  int nst;            // shared-memory ring stages of the core kernel
  size_t core_smem;   // dynamic shared memory of the core kernel
  int Kg, Kgp;        // output-projection K (2F or 3F) and padded
  int ntile_out;      // output-projection N tile (<= 256)
  int gemm_nst;
  size_t gemm_smem;
  // workspace byte offsets
  size_t off_Q, off_KH, off_VH, off_Z, off_kvec, off_qvec, off_orig, off_flag;
  size_t off_O, off_W, off_stats, off_feat, off_wT, off_rowflag, total;
};

// Returns 0 and fills `p`, or a nonzero reason code: 1 = bad dims, 2 = unsupported.
static inline int make_plan(Plan& p, int B, int N, int H, int D, int Dv, int P, int Q, int Cz, int R,
                            int Cout, int f32, const char** why) {
  *why = "";
  if (B <= 0 || N <= 0 || H <= 0 || D <= 0 || Dv <= 0 || P <= 0 || Q <= 0 || Cz <= 0 || R <= 0 ||
      Cout <= 0) {
    *why = "every dimension must be positive";
    return 1;
  }
  p.B = B; p.N = N; p.H = H; p.D = D; p.Dv = Dv; p.P = P; p.Q = Q; p.Cz = Cz; p.R = R; p.Cout = Cout;
  p.F = H * (Dv + 4 * Q + Cz);
  p.f32 = f32 ? 1 : 0;
  p.nT = cdiv(N, kTile);
  p.nsq = f32 ? 3 : 1;
  p.nsv = f32 ? 2 : 1;
  p.nz = f32 ? 3 : 1;
  p.nzv = f32 ? 2 : 1;
  p.KHc = p.nsq * D + 9 * P;
  p.KHp = rup(p.KHc, kChunk);
  p.nKH = p.KHp / kChunk;
  p.Zc = p.nz * R * Cz;
  p.Zp = rup(p.Zc, kChunk);
  p.nZ = p.Zp / kChunk;
  p.Kq = p.KHp + p.Zp;
  p.nQc = p.Kq / kChunk;
  p.VHc = p.nsv * Dv + 6 * Q;
  p.VHp = rup(p.VHc, kChunk);
  p.nVH = p.VHp / kChunk;
  p.ZVc = p.nzv * R * Cz;
  p.nZV = cdiv(p.ZVc, kChunk);
  p.Ocols = p.VHp + p.nZV * kChunk;
  p.Pcols = f32 ? 128 : 64;
  p.tmemO = kTmemP + p.Pcols;
  if (p.nT > kMaxTiles) { *why = "N above 262144 is not supported"; return 2; }
  if (P > kMaxPts || Q > kMaxPts) { *why = "more than 64 points per head is not supported"; return 2; }
  if (R * Cz > kMaxRCz) { *why = "R*Cz above 1024 is not supported"; return 2; }
  if (p.nQc > kMaxQChunks) { *why = "lifted query width above 512 columns is not supported"; return 2; }
  if (p.tmemO + p.Ocols > 512) { *why = "lifted value width exceeds the 512 tensor-memory columns"; return 2; }
  // core shared memory: resident Qhat + ring + barriers/buffers (+1 KB alignment slack)
  const size_t fixed = 1024 + 4096 + 2 * kMaxTiles;
  const size_t limit = 232448;  // 227 KB opt-in maximum per block on sm_100
  size_t avail = limit - fixed - (size_t)p.nQc * 16384;
  int nst = (int)(avail / 16384);
  if (nst > 8) nst = 8;
  if (nst < 3) { *why = "shared memory too small for the ring"; return 2; }
  p.nst = nst;
  p.core_smem = fixed + (size_t)(p.nQc + nst) * 16384;
  if (p.core_smem < 120 * 1024) p.core_smem = 120 * 1024;   // one CTA per SM (TMEM is taken whole)
  // output projection
  p.Kg = (f32 ? 3 : 2) * p.F;
  p.Kgp = rup(p.Kg, kChunk);
  p.ntile_out = Cout >= 256 ? 256 : rup(Cout, 16);
  {
    size_t stage = 16384 + (size_t)p.ntile_out * 128;
    int g = (int)((limit - 2048) / stage);
    p.gemm_nst = g > 4 ? 4 : g;
    p.gemm_smem = 2048 + stage * p.gemm_nst;
  }
  // workspace layout
  const size_t BN = (size_t)B * N, BHN = (size_t)B * H * N;
  size_t o = 0;
  auto take = [&](size_t bytes) { size_t at = o; o = rup_sz(o + bytes, 256); return at; };
  p.off_Q = take(BHN * p.Kq * 2);
  p.off_KH = take(BHN * p.KHp * 2);
  p.off_VH = take(BHN * p.VHp * 2);
  p.off_Z = take(BN * p.Zp * 2);
  p.off_kvec = take(BHN * 16);
  p.off_qvec = take(BHN * 16);
  p.off_orig = take((size_t)B * p.nT * 16);
  p.off_flag = take((size_t)B * p.nT * 4);
  p.off_O = take(BN * H * p.Ocols * 4);
  p.off_W = take(BN * H * 16);
  p.off_stats = take(BHN * 8);
  p.off_feat = take(BN * p.Kgp * 2);
  p.off_wT = take((size_t)rup(Cout, p.ntile_out) * p.Kgp * 2);
  p.off_rowflag = take(BN);
  p.total = o;
  return 0;
}

}  // namespace fipa
