// bwd_plan.h -- sizes and workspace layout of the backward pass of the fused
// IPA core (training), appended after the forward's workspace (plan.h).
//
// The backward recomputes the forward (lift and fused core, the core also
// saving the normalised aggregates O of every row), then:
//   dfeat  = d_update @ w_out^T              (tcgen05, bfloat16 hi/lo parts)
//   prep   per residue: dO = [d o_scalar | dG | dG | dU], D = dO . O, the
//          frame and pair-value parts of the chain rule, fp32 features
//   q-side per (query tile, head): S and dP recomputed on tcgen05, dS =
//          P (dP - D), dQhat = dS . [k | b' | z2] in tensor memory
//   k-side per (key tile, head): S^T and dP^T recomputed, dKhat = dS^T Qhat,
//          dVhat = P^T dO and dz2 = dS^T u + P^T dU in tensor memory
//   chain  per residue: points through the frames, z1 / z2 / Wb / point
//          weights, deterministic partial sums
//   dw_out = features^T d_update, db_out     (tcgen05, bfloat16 hi/lo parts)
#pragma once

#include "plan.h"

namespace fipa {

struct BwdPlan {
  int Osw;        // saved aggregate row: Dv + 3Q + R*Cz floats
  int Vw;         // dO row width (fp16 columns): VHp + nZ * 64, the value-operand width
  int nOc;        // dO chunks (nVH + nZ)
  int nQr;        // q-side resident Qhat chunks: head part + u hi (nKH + nZ)
  int q_nst;      // q-side ring stages
  size_t q_smem;
  int tmDS, tmDQ; // q-side TMEM columns of dS (fp16 pairs) and of the dQhat accumulator
  int k_nres;     // k-side resident key chunks: KH + Z + VH
  int k_nst;
  size_t k_smem;
  int tmDK, tmDV, tmDZ;   // k-side TMEM columns of the accumulators
  int Kr;         // q-side result row: [sum dS k (D) | X (3P) | rs | W (3) | E], padded to 4
  int Kk;         // k-side result row: [sum dS q/sqrt(3D) (D) | 2g Y (3P) | cs | V (3) | dv (Dv) | dg (3Q)], padded to 4
  int Fp;         // feature row [F features | 1 | pad], padded to 64 (bfloat16 hi and lo copies)
  int Coutp;      // Cout padded to 64: row width of the bfloat16 copies of d_update and w_out
  int RCz;
  int chain_res;  // residues per chain CTA
  int nchain;     // chain CTAs
  int dw_ks;      // row splits of the dw_out GEMM
  size_t off_lp, off_osave, off_dfeat, off_fhi, off_flo, off_duhi, off_dulo, off_whi, off_wlo, off_dO, off_dvec,
      off_rloc, off_dz1u;
  size_t off_qres, off_du, off_kres, off_dz2h, off_dwpart, off_wbpart, off_gpart, total;
};

constexpr int kBwdTailQ = 8192;    // q-side kernel: barriers, key terms, tile list
constexpr int kBwdTailK = 16384;   // k-side kernel: barriers, per-query data, tile list
constexpr int kChainRes = 32;

// Returns 0, or 2 (unsupported) with a reason.  `p` is the forward plan of
// the same dims (bfloat16 inputs).
static inline int make_bwd_plan(BwdPlan& b, const Plan& p, const char** why) {
  *why = "";
  if (p.f32) { *why = "the backward pass supports bfloat16 inputs only"; return 2; }
  b.RCz = p.R * p.Cz;
  b.Osw = p.Dv + 3 * p.Q + b.RCz;
  b.nOc = p.nVH + p.nZ;
  b.Vw = b.nOc * kChunk;
  b.nQr = p.nKH + p.nZ;
  // tensor memory: q side S/dP (128) + dS (64) + dQhat (64 per K chunk)
  b.tmDS = 128;
  b.tmDQ = 192;
  if (b.tmDQ + 64 * b.nQr > 512) { *why = "backward: lifted key width exceeds the tensor-memory budget"; return 2; }
  // k side S^T/dP^T (128) + dK head (64 nKH) + dV head (64 nVH) + dz2 (64 nZ)
  b.tmDK = 128;
  b.tmDV = b.tmDK + 64 * p.nKH;
  b.tmDZ = b.tmDV + 64 * p.nVH;
  if (b.tmDZ + 64 * p.nZ > 512) { *why = "backward: lifted widths exceed the tensor-memory budget"; return 2; }
  const size_t limit = 232448, slack = 1024;
  {
    const long left = (long)limit - (long)slack - kBwdTailQ - (long)(b.nQr + b.nOc) * 16384;
    int nst = (int)(left / 16384);
    if (nst > 8) nst = 8;
    if (nst > p.ring_cap) nst = p.ring_cap;
    if (nst < 2) { *why = "backward: shared memory too small for the q-side ring"; return 2; }
    b.q_nst = nst;
    b.q_smem = slack + kBwdTailQ + (size_t)(b.nQr + b.nOc + nst) * 16384;
  }
  {
    b.k_nres = p.nKH + p.nZ + p.nVH;
    const long left = (long)limit - (long)slack - kBwdTailK - (long)(b.k_nres + 4) * 16384;
    int nst = (int)(left / 16384);
    if (nst > 8) nst = 8;
    if (nst > p.ring_cap) nst = p.ring_cap;
    if (nst < 2) { *why = "backward: shared memory too small for the k-side ring"; return 2; }
    b.k_nst = nst;
    b.k_smem = slack + kBwdTailK + (size_t)(b.k_nres + 4 + nst) * 16384;
  }
  b.Kr = rup(p.D + 3 * p.P + 5, 4);
  b.Kk = rup(p.D + 3 * p.P + 4 + p.Dv + 3 * p.Q, 4);
  b.Fp = rup(p.F + 1, 64);
  b.Coutp = rup(p.Cout, 64);
  b.chain_res = kChainRes;
  const int BN = p.B * p.N;
  b.nchain = cdiv(BN, kChainRes);
  {
    // one wave of the dw_out GEMM's 128 x 256 tiles, split over 64-row chunks
    const int tiles = cdiv(b.Fp, 128) * cdiv(p.Cout, 256);
    int ks = cdiv(148, tiles);
    const int maxks = cdiv(BN, 64);
    if (ks > maxks) ks = maxks;
    if (ks < 1) ks = 1;
    b.dw_ks = ks;
  }
  const size_t BNs = (size_t)BN, BHN = (size_t)p.B * p.H * p.N;
  size_t o = rup_sz(p.total, 256);
  auto take = [&](size_t bytes) { size_t at = o; o = rup_sz(o + bytes, 256); return at; };
  b.off_lp = take(BHN * 3 * p.Q * 4);          // local points of the recompute (not an output)
  b.off_osave = take(BHN * b.Osw * 4);
  b.off_dfeat = take(BNs * p.F * 4);
  b.off_fhi = take(BNs * b.Fp * 2);
  b.off_flo = take(BNs * b.Fp * 2);
  b.off_duhi = take(BNs * b.Coutp * 2);
  b.off_dulo = take(BNs * b.Coutp * 2);
  b.off_whi = take((size_t)p.F * b.Coutp * 2);
  b.off_wlo = take((size_t)p.F * b.Coutp * 2);
  b.off_dO = take(BHN * b.Vw * 2);
  b.off_dvec = take(BHN * 16);
  b.off_rloc = take(BNs * 12 * 4);
  b.off_dz1u = take(BNs * b.RCz * 4);
  b.off_qres = take(BHN * b.Kr * 4);
  b.off_du = take(BHN * b.RCz * 4);
  b.off_kres = take(BHN * b.Kk * 4);
  b.off_dz2h = take(BHN * b.RCz * 4);
  b.off_dwpart = take((size_t)b.dw_ks * b.Fp * p.Cout * 4);
  b.off_wbpart = take((size_t)b.nchain * p.Cz * p.H * 4);
  b.off_gpart = take((size_t)b.nchain * p.H * 4);
  b.total = o;
  return 0;
}

}  // namespace fipa
