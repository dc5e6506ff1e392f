// plan.h -- derived sizes and device-workspace layout of one fused IPA forward.
//
// Lifted operand layout (FlashIPA, "Flash Invariant Point Attention": the
// squared-norm expansion |a-b|^2 = |a|^2 - 2 a.b + |b|^2 turns the point
// term into a dot product; the pair factors z1, z2 turn the pair bias and the
// pair aggregation into dot products).  Rows are fp16; a value that needs
// more than 11 significant bits is stored as hi + lo halves.
//
// bfloat16 inputs (the point term runs on the tensor cores):
//   Qhat [B*H, N, Kq] = [ QH (KHp) | u hi (Zp) | u lo (Zp) ]
//       QH = [ q/sqrt(3D) | 2g a' hi | 2g a' hi | 2g a' lo | 0.. ],  u = z1[r,c] Wb[c,h]/sqrt(3)
//   KH   [B*H, N, KHp] = [ k | b' hi | b' lo | b' hi | 0.. ]
//   Z    [B,   N, Zp ] = [ z2 ]          (exact in fp16; multiplies both u halves)
//   VH   [B*H, N, VHp] = [ v | g' hi | g' lo | 0.. ]
// float32 inputs (every value split, the point term in fp32 on the CUDA cores):
//   QH = [ q/sqrt(3D) hi | hi | lo | 0.. ],  KH = [ k hi | lo | hi | 0.. ]
//   Qhat pair part = [ u hi | u hi | u lo ],  Z = [ z2 hi | z2 lo | z2 hi ]
//   VH = [ v hi | v lo | g' hi | g' lo | 0.. ]
//   QP, KP [B*H, N, 3P] fp32: a' and b' for the exact squared distance
// where a' = T_i(q_p) - o_G, b' = T_j(k_p) - o_G, g' = T_j(v_q) - o_G are
// global points relative to the mean translation o_G of the residue's own
// 32-residue group, and g is the per-head distance weight.  Every column
// segment is padded to a multiple of 8 columns.  The value product uses the
// first ZV columns of Z (f32: z2 hi | z2 lo).
#pragma once

#include <stddef.h>
#include <stdint.h>

namespace fipa {

constexpr int kTile = 128;       // residues per query / key tile (MMA M and N)
constexpr int kGroup = 32;       // residues sharing one coordinate origin (4 groups per tile)
constexpr int kChunk = 64;       // fp16 columns per 128-byte swizzled chunk
constexpr int kTmemS = 0;        // TMEM column of the logit tile S (128 fp32 columns)
constexpr int kTmemP = 128;      // TMEM column of P (fp16 pairs: 64 columns, 128 when split)
constexpr int kMaxQChunks = 10;  // resident Qhat tile <= 160 KB of shared memory
constexpr int kVbufMinTiles = 8;  // key tiles from which the value-buffer mode pays
constexpr int kMaxPts = 64;      // points per head handled by the prologue scratch
constexpr int kMaxRCz = 1024;    // R*Cz handled by the prologue scratch
constexpr int kMaxTiles = 1024;  // key tiles per sample (N <= 131072)
constexpr int kOaccTiles = 4;    // float32 inputs: key tiles per tensor-memory segment of O
constexpr int kMaxPSimt = 16;    // points per head of the fp32 (exact distance) mode
constexpr int kLiftRes = 8;      // most residues per prologue lift CTA (divides the 32-residue group)
constexpr int kWpTiles = 4;      // 32x32 output-weight tiles per weight-preparation CTA

#ifdef __CUDACC__
#define FIPA_HD __host__ __device__
#else
#define FIPA_HD
#endif

FIPA_HD static inline int cdiv(int a, int b) { return (a + b - 1) / b; }

// Division by an invariant divisor d >= 1 as one wide multiply and a shift
// (Granlund and Montgomery, "Division by invariant integers using
// multiplication", 1994): with l = ceil(log2 d), p = 31 + l and
// m = ceil(2^p / d) (< 2^32), floor(n / d) = floor(n * m / 2^p) for every
// 0 <= n < 2^31, because m = (2^p + e) / d with 0 <= e < d adds less than
// n e / (d 2^p) < 2^-l <= 1/d to n / d, which never reaches the next integer.
struct FastDiv {
  uint32_t d, m, p;
  FIPA_HD uint32_t div(uint32_t n) const { return (uint32_t)(((uint64_t)n * m) >> p); }
};
static inline FastDiv make_fastdiv(uint32_t d) {
  uint32_t l = 0;
  while ((1ull << l) < d) ++l;
  const uint32_t p = 31 + l;
  return FastDiv{d, (uint32_t)(((1ull << p) + d - 1) / d), p};
}
FIPA_HD static inline int rup(int a, int b) { return cdiv(a, b) * b; }
static inline size_t rup_sz(size_t a, size_t b) { return (a + b - 1) / b * b; }

struct Plan {
  int B, N, H, D, Dv, P, Q, Cz, R, Cout, F;
  int f32;            // 1: float32 layout (hi/lo splits everywhere, fp32 distance); 0: bfloat16 layout
  int in_f32;         // dtype of the inputs: 1 float32, 0 bfloat16 (== f32, except for the backward's
                      // recompute of float32 inputs in the bfloat16 layout)
  int nT;             // tiles per sample
  // query rows computed by this forward, the same range in every sample: row0
  // a multiple of the 128-row tile, row1 a multiple of it or N (all keys are
  // still lifted; rows outside the range are left untouched in the outputs)
  int row0, row1;
  int nG;             // 32-residue origin groups per sample (4 per tile)
  int nsq;            // copies of the scalar q/k columns (1 or 3)
  int nsv;            // copies of the scalar v columns (1 or 2)
  int nz;             // copies of the pair columns on the key side (1 or 3)
  int nzv;            // copies of the pair columns on the value side (1 or 2)
  int KHc, KHp, nKH;  // key/query head-part columns, padded, chunks
  int Zc, Zp, nZ;     // pair columns, padded, chunks
  int nqz;            // Qhat chunks multiplying each Z chunk (2: u hi and u lo)
  int D8, P38, Dv8, Q38, RC8;  // segment widths, each padded to 8 columns (one 16-byte chunk)
  int geo_simt;       // 1: squared distance in fp32 on the CUDA cores (f32 inputs)
  int Kq, nQc;        // Qhat row width and chunks
  int VHc, VHp, nVH;  // value head-part columns, padded, chunks
  int ones_col;       // float32 inputs: value column holding 1 (the P.V product's own sum of P), or -1
  int oacc_T;         // float32 inputs: key tiles per tensor-memory segment of O (0 = one segment)
  int oacc_off;       // tail offset of the per-row fp32 accumulator [128][Ocols + 1] (oacc_T > 0)
  int ZVc, nZV;       // pair columns used by the value product, chunks
  int Ocols;          // VHp + nZV * 64: fp32 accumulator columns per row
  int Pcols;          // TMEM columns holding P (64, or 128 for hi+lo)
  int tmemO;          // TMEM column of the O accumulator
  int nst;            // shared-memory ring stages of the core kernel
  int ring_cap;       // most ring stages any kernel of this plan may use (tuning; default 8)
  // Value-buffer mode (bfloat16 inputs, when it fits): only QH and u hi of the
  // Qhat tile stay resident, the u lo chunks stream through the ring with the
  // key chunks, and each key tile's value chunks [VH | Z] land in a buffer of
  // their own, so every P.V product runs over contiguous 64-column groups.
  int vbuf;           // 1: value-buffer mode
  int nQres;          // resident Qhat chunks (nQc, or nKH + nZ in value-buffer mode)
  int nVB;            // value chunks per key tile (nVH + nZV); buffered in value-buffer mode
  size_t core_smem;   // dynamic shared memory of the core kernel
  size_t lift_smem;   // dynamic shared memory of the prologue lift kernel
  FastDiv fd_H, fd_P, fd_Q, fd_Cz;               // divisors of the lift kernel's index maps
  FastDiv fd_nQ8, fd_nK8, fd_nV8, fd_nZ8;        // 16-byte chunks per lifted row type
  FastDiv fd_nQ8e;    // Qhat chunks the lift iterates per row (a u-hi chunk also writes its lo partner)
  FastDiv fd_D8v, fd_Dv8v, fd_RC8v;              // 8-value vectors per staged row
  // Output-projection operand: one block per head, in head order, each block
  // nseg segments (bf16: [hi | lo], f32: [hi | hi | lo]) of Wh8 columns holding
  // [scalar (Dv) | x (Q) | y (Q) | z (Q) | lengths (Q) | pair (Cz) | pad].  The
  // projection's sum over k is taken in this order; the weights are permuted
  // to match, so the result is features @ w_out in the page's feature order.
  int Wh, Wh8, nseg;  // head-block feature width, padded to 8, segments
  int Kg, Kgp;        // output-projection K (H * nseg * Wh8) and padded
  int ntile_out;      // output-projection N tile (<= 256)
  int gemm_ks;        // output-projection split-K factor
  int gemm_nks;       // K chunks per split
  int gemm_nst;
  size_t gemm_smem;
  int wp_ctas;        // weight-preparation CTAs at the front of the prologue launch
  int lift_res;       // residues per lift CTA: 4 when that grid still fits about one resident wave, else 8
  int lift_ctas;      // lift CTAs per sample (lift_res residues each)
  // workspace byte offsets
  size_t off_Q, off_KH, off_VH, off_Z, off_kvec, off_qvec, off_orig, off_flag;
  size_t off_QP, off_KP;
  size_t off_stats, off_feat, off_wT, off_rowflag, total;
};

// Returns 0 and fills `p`, or a nonzero reason code: 1 = bad dims, 2 = unsupported.
// pair_split: 1 = pair-bias operand as fp16 hi + lo halves (bfloat16 inputs);
// 0 = hi half only.  value_buffer: 1 = value-buffer mode where it fits and the
// sample spans at least kVbufMinTiles key tiles, 2 = wherever it fits, 0 = off.
static inline int make_plan(Plan& p, int B, int N, int H, int D, int Dv, int P, int Q, int Cz, int R,
                            int Cout, int f32, const char** why, int pair_split = 1, int value_buffer = 1,
                            int ring_cap = 8) {
  *why = "";
  if (B <= 0 || N <= 0 || H <= 0 || D <= 0 || Dv <= 0 || P <= 0 || Q <= 0 || Cz <= 0 || R <= 0 ||
      Cout <= 0) {
    *why = "every dimension must be positive";
    return 1;
  }
  p.B = B; p.N = N; p.H = H; p.D = D; p.Dv = Dv; p.P = P; p.Q = Q; p.Cz = Cz; p.R = R; p.Cout = Cout;
  p.F = H * (Dv + 4 * Q + Cz);
  p.f32 = f32 ? 1 : 0;
  p.in_f32 = p.f32;
  p.nT = cdiv(N, kTile);
  p.row0 = 0;
  p.row1 = N;
  p.nG = 4 * p.nT;
  p.nsq = f32 ? 3 : 1;
  p.nsv = f32 ? 2 : 1;
  p.nz = f32 ? 3 : 1;
  p.nzv = f32 ? 2 : 1;
  p.nqz = f32 ? 1 : (pair_split ? 2 : 1);
  p.geo_simt = f32 ? 1 : 0;
  p.D8 = rup(D, 8);
  p.P38 = rup(3 * P, 8);
  p.Dv8 = rup(Dv, 8);
  p.Q38 = rup(3 * Q, 8);
  p.RC8 = rup(R * Cz, 8);
  p.KHc = p.nsq * p.D8 + (p.geo_simt ? 0 : 3 * p.P38);
  p.KHp = rup(p.KHc, kChunk);
  p.nKH = p.KHp / kChunk;
  p.Zc = p.nz * p.RC8;
  p.Zp = rup(p.Zc, kChunk);
  p.nZ = p.Zp / kChunk;
  p.Kq = p.KHp + p.nqz * p.Zp;
  p.nQc = p.Kq / kChunk;
  p.VHc = p.nsv * p.Dv8 + 2 * p.Q38;
  p.VHp = rup(p.VHc, kChunk);
  p.ones_col = (f32 && p.VHp > p.VHc) ? p.VHc : -1;
  p.nVH = p.VHp / kChunk;
  p.ZVc = p.nzv * p.RC8;
  p.nZV = cdiv(p.ZVc, kChunk);
  p.Ocols = p.VHp + p.nZV * kChunk;
  p.Pcols = f32 ? 128 : 64;
  p.tmemO = kTmemP + p.Pcols;
  if (p.nT > kMaxTiles) { *why = "N above 131072 is not supported"; return 2; }
  if (p.geo_simt && P > kMaxPSimt) { *why = "more than 16 points per head with float32 inputs is not supported"; return 2; }
  if (P > kMaxPts || Q > kMaxPts) { *why = "more than 64 points per head is not supported"; return 2; }
  if (H > 64) { *why = "more than 64 heads is not supported"; return 2; }
  if (R * Cz > kMaxRCz) { *why = "R*Cz above 1024 is not supported"; return 2; }
  if (p.nQc > kMaxQChunks) { *why = "lifted query width above 640 columns is not supported"; return 2; }
  if (p.tmemO + p.Ocols > 512) { *why = "lifted value width exceeds the 512 tensor-memory columns"; return 2; }
  // core shared memory: resident Qhat + ring + barriers/buffers (+1 KB alignment slack)
  const size_t kp_bytes = p.geo_simt ? (size_t)2 * kTile * 3 * P * 4 : 0;
  size_t fixed = 1024 + 5120 + 2 * kMaxTiles + kp_bytes;   // slack + tail (see core.cu)
  const size_t limit = 232448;  // 227 KB opt-in maximum per block on sm_100
  // float32 inputs: the tensor cores accumulate O for kOaccTiles key tiles at a
  // time, then the softmax warps add it into a per-row fp32 accumulator (round
  // to nearest) in the tail, so no fp32 sum in tensor memory spans more than
  // 16 x kOaccTiles key slices (its rounding drifts with the number of terms)
  p.oacc_T = 0;
  p.oacc_off = 0;
  if (f32) {
    const size_t oacc_bytes = (size_t)kTile * (p.Ocols + 1) * 4;
    const size_t need = limit - (fixed + oacc_bytes) - (size_t)p.nQc * 16384;
    if (fixed + oacc_bytes + (size_t)p.nQc * 16384 < limit && need / 16384 >= 3) {
      p.oacc_T = kOaccTiles;
      p.oacc_off = (int)(5120 + 2 * kMaxTiles + kp_bytes);
      fixed += oacc_bytes;
    }
  }
  p.nVB = p.nVH + p.nZV;
  p.vbuf = 0;
  p.nQres = p.nQc;
  // Measured on B200: 2-6% faster on the core from N = 2048 up; about 1% slower
  // with two key tiles, where the serialised value loads are not hidden.
  const bool vb_len = value_buffer == 2 || cdiv(N, kTile) >= kVbufMinTiles;
  if (value_buffer && vb_len && p.nqz == 2 && !p.geo_simt) {
    const int nres = p.nKH + p.nZ;
    const long left = (long)limit - (long)fixed - (long)(nres + p.nVB) * 16384;
    if (left >= 3 * 16384) { p.vbuf = 1; p.nQres = nres; }
  }
  size_t avail = limit - fixed - (size_t)(p.nQres + (p.vbuf ? p.nVB : 0)) * 16384;
  int nst = (int)(avail / 16384);
  if (nst > 8) nst = 8;
  if (nst > ring_cap) nst = ring_cap;
  p.ring_cap = ring_cap;
  if (nst < 2 || (nst < 3 && ring_cap >= 3)) { *why = "shared memory too small for the ring"; return 2; }
  p.nst = nst;
  const int nchunks = p.nQres + (p.vbuf ? p.nVB : 0) + nst;   // Qhat, value buffer, ring
  p.core_smem = fixed + (size_t)nchunks * 16384;
  if (p.core_smem < 120 * 1024) p.core_smem = 120 * 1024;   // one CTA per SM (TMEM is taken whole)
  if (p.oacc_T == 0 && (size_t)kTile * (p.Ocols + 1) * 4 > (size_t)nchunks * 16384) {
    *why = "value width too large for the epilogue staging"; return 2;
  }
  // prologue lift kernel: Wb^T, zero-padded z1 / q / k / v / point rows
  // and frames of lift_res residues, and the chunk table of the four row types
  p.lift_res = (size_t)B * cdiv(N, 4) <= 148 * 6 ? 4 : kLiftRes;
  p.lift_smem = ((size_t)rup(H * Cz, 8) + (size_t)p.lift_res * p.RC8 +
                 (size_t)p.lift_res * H * (2 * p.D8 + p.Dv8 + 2 * p.P38 + p.Q38) + p.lift_res * 12) * 4 +
                (size_t)(p.Kq + p.KHp + p.VHp + p.Zp) / 8 * 4;
  p.fd_H = make_fastdiv(H); p.fd_P = make_fastdiv(P); p.fd_Q = make_fastdiv(Q); p.fd_Cz = make_fastdiv(Cz);
  p.fd_nQ8 = make_fastdiv(p.Kq / 8); p.fd_nK8 = make_fastdiv(p.KHp / 8);
  p.fd_nQ8e = make_fastdiv(p.nqz == 2 ? (p.KHp + p.Zp) / 8 : p.Kq / 8);
  p.fd_nV8 = make_fastdiv(p.VHp / 8); p.fd_nZ8 = make_fastdiv(p.Zp / 8);
  p.fd_D8v = make_fastdiv(p.D8 / 8); p.fd_Dv8v = make_fastdiv(p.Dv8 / 8); p.fd_RC8v = make_fastdiv(p.RC8 / 8);
  if (p.lift_smem > 160 * 1024) { *why = "prologue staging exceeds shared memory (H*Cz or R*Cz too large)"; return 2; }
  // output projection
  p.Wh = Dv + 4 * Q + Cz;
  p.Wh8 = rup(p.Wh, 8);
  p.nseg = f32 ? 3 : 2;
  p.Kg = H * p.nseg * p.Wh8;
  p.Kgp = rup(p.Kg, kChunk);
  // N tile and split-K so that the grid covers the SMs (deterministic split-K:
  // the splits of an output tile form one thread-block cluster and add their
  // partial tiles in split order through distributed shared memory)
  {
    // N tile = all of Cout up to 256 (wide MMAs); split-K fills the SMs
    const int mt = cdiv(B * N, kTile), nk = p.Kgp / kChunk;
    const int nt_w = Cout >= 256 ? 256 : rup(Cout, 16);
    p.ntile_out = nt_w;
    const int tiles = mt * cdiv(Cout, nt_w);
    // split-K factor: fill the SMs, at least 4 K chunks per split, and at most
    // 8 splits (the splits of a tile form one portable-size cluster)
    int ks = tiles >= 148 ? 1 : cdiv(148, tiles);
    if (ks > nk / 4) ks = nk / 4 > 1 ? nk / 4 : 1;
    if (ks > 8) ks = 8;
    p.gemm_nks = cdiv(nk, ks);
    p.gemm_ks = cdiv(nk, p.gemm_nks);
    size_t stage = 16384 + (size_t)p.ntile_out * 128;
    int g = (int)((limit - 2048) / stage);
    p.gemm_nst = g > 8 ? 8 : g;
    p.gemm_smem = 2048 + stage * p.gemm_nst;
  }
  p.wp_ctas = cdiv(cdiv(p.F, 32) * cdiv(rup(Cout, p.ntile_out), 32), kWpTiles);
  p.lift_ctas = cdiv(N, p.lift_res);
  if (p.lift_smem < 32 * 33 * 4) p.lift_smem = 32 * 33 * 4;   // the weight-prep tile
  // workspace layout
  const size_t BN = (size_t)B * N, BHN = (size_t)B * H * N;
  size_t o = 0;
  auto take = [&](size_t bytes) { size_t at = o; o = rup_sz(o + bytes, 256); return at; };
  p.off_Q = take(BHN * p.Kq * 2);
  p.off_KH = take(BHN * p.KHp * 2);
  p.off_VH = take(BHN * p.VHp * 2);
  p.off_Z = take(BN * p.Zp * 2);
  p.off_QP = take(p.geo_simt ? BHN * 3 * P * 4 : 0);
  p.off_KP = take(p.geo_simt ? BHN * 3 * P * 4 : 0);
  p.off_kvec = take(BHN * 16);
  p.off_qvec = take(BHN * 16);
  p.off_orig = take((size_t)B * p.nG * 16);
  p.off_flag = take((size_t)B * p.nT * 4);
  p.off_stats = take(BHN * 8);
  p.off_feat = take(BN * p.Kgp * 2);
  p.off_wT = take((size_t)rup(Cout, p.ntile_out) * p.Kgp * 2);
  p.off_rowflag = take(BN);
  p.total = o;
  return 0;
}

}  // namespace fipa
