// core.cu -- fused flash-style IPA attention on tcgen05 tensor cores.
//
// One CTA per (128-row query tile, head, sample).  No N x N tensor leaves the
// SM: the logit tile S = Qhat Khat^T (lifted columns, see plan.h) accumulates
// in tensor memory, four softmax warps finish the logits in fp32 (per-key and
// per-row origin corrections, masks), run an online softmax with a lazily
// updated running max, and write P as fp16 back into tensor memory, where the
// next tcgen05.mma consumes it as the A operand of O += P [v | g' | z2].
//
// The logit (page "Invariant point attention (IPA)", Required behavior) is
//   L_ij = q.k/sqrt(3D) + bias_ij/sqrt(3) - g sum_p |a_p - b_p|^2,
// and with tile origins o_q, o_k, a' = a - o_q, b' = b - o_k, D = o_q - o_k:
//   -g sum|a-b|^2 = -g sum|a'|^2 - g sum|b'|^2 + 2g sum a'.b'
//                   - g P |D|^2 - 2g D.sum a' + 2g D.sum b'.
// 2g a'.b' runs on the tensor cores (hi/lo fp16 halves); -g sum|b'|^2 + 2g D.sum b'
// is a per-key fp32 term, -g P|D|^2 - 2g D.sum a' a per-row fp32 term, and the
// per-row -g sum|a'|^2 cancels in the softmax (it is added back only for lse).
//
// Warp roles (256 threads):
//   warp 0      TMA producer: resident Qhat tile, then a ring of 16 KB chunks
//   warp 1      tcgen05.mma issuer (single thread) and TMEM owner
//   warps 2-3   per-key fp32 terms of each key tile, into shared memory
//   warps 4-7   softmax: one thread per query row = one TMEM lane
#include "kernels.h"
#include "sm100.cuh"

namespace fipa {
namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kTau = 8.0f;   // rescale O only when the row max grows by more than 2^8

struct CoreArgs {
  Plan p;
  const float4* kvec;
  const float4* qvec;
  const float* QP;
  const float* KP;
  const float4* orig;
  const int* flag;
  const uint8_t* mask;
  const uint8_t* pair_mask;
  const void* raw;
  const void* rot;
  const void* trans;
  const void* z1;
  __half* feat;
  uint8_t* rowflag;
  float* local_points;
  float eps;
  float2* stats;
  float* lse;
  int* status;
  unsigned long long timeout_ns;
  long long* trace;
  int trace_cta;
  // training recompute only (SAVE instantiation): normalised aggregates of
  // every (residue, head), [B*N*H, Dv + 3Q + R*Cz] fp32 = [o_scalar | G (global
  // value points, xyz per point) | U = sum_j a_ij z2_j], for the backward pass
  float* osave;
};

// Shared-memory tail after the Qhat tile and the ring (byte offsets).
constexpr int kBarFull = 0;        // 8 x u64
constexpr int kBarEmpty = 64;      // 8 x u64
constexpr int kBarQ = 128;
constexpr int kBarSFull = 136;
constexpr int kBarSFree = 144;
constexpr int kBarPFull = 152;
constexpr int kBarPVDone = 160;
constexpr int kBarKtFull = 168;    // 2 x u64
constexpr int kBarKtEmpty = 184;   // 2 x u64
constexpr int kBarDrain = 200;
constexpr int kBarVFull = 208;      // value buffer of the current key tile landed (value-buffer mode)
constexpr int kOkBuf = 256;        // 2 x 4 key-group origins (float4)
constexpr int kMisc = 384;         // tmem slot, abort flag, tile count
constexpr int kKtBuf = 1024;       // 2 x 4 query groups x 128 keys per-key terms (floats)
constexpr int kTiles = 5120;       // uint16 key-tile list (<= 1024 entries)
constexpr int kKpBuf = 7168;       // fp32 key points of two key tiles (float32-input mode)

__device__ __forceinline__ float load_raw(const CoreArgs& a, int h) {
  return a.p.in_f32 ? static_cast<const float*>(a.raw)[h]
                 : __bfloat162float(static_cast<const __nv_bfloat16*>(a.raw)[h]);
}

__device__ __forceinline__ float ld_any(const void* ptr, size_t i, int f32) {
  return f32 ? __ldg(static_cast<const float*>(ptr) + i)
             : __bfloat162float(static_cast<const __nv_bfloat16*>(ptr)[i]);
}


// 8 feature values at columns [c, c+8) of one head block of the projection
// operand: fp16 hi at c and the residual lo = fp16(x - hi) at F+c, F the
// segment stride (float32 inputs: hi, hi, lo at c, F+c, 2F+c); n <= 8 of them
// are stored.  One 16-byte store per segment where the run is aligned.
__device__ __forceinline__ void put8(__half* frow, int F, int f32, int c, int n, const float (&v)[8]) {
  uint32_t hw[4], lw[4];
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    const __half2 h = __floats2half2_rn(v[2 * t], v[2 * t + 1]);
    const float2 f = __half22float2(h);
    const __half2 l = __floats2half2_rn(v[2 * t] - f.x, v[2 * t + 1] - f.y);
    hw[t] = *reinterpret_cast<const uint32_t*>(&h);
    lw[t] = *reinterpret_cast<const uint32_t*>(&l);
  }
  if (n == 8 && ((c | F) & 7) == 0) {
    const uint4 H4 = make_uint4(hw[0], hw[1], hw[2], hw[3]), L4 = make_uint4(lw[0], lw[1], lw[2], lw[3]);
    *reinterpret_cast<uint4*>(frow + c) = H4;
    if (f32) {
      *reinterpret_cast<uint4*>(frow + F + c) = H4;
      *reinterpret_cast<uint4*>(frow + 2 * F + c) = L4;
    } else {
      *reinterpret_cast<uint4*>(frow + F + c) = L4;
    }
  } else {
    const __half* hh = reinterpret_cast<const __half*>(hw);
    const __half* ll = reinterpret_cast<const __half*>(lw);
    for (int t = 0; t < n; ++t) {
      frow[c + t] = hh[t];
      if (f32) { frow[F + c + t] = hh[t]; frow[2 * F + c + t] = ll[t]; }
      else     { frow[F + c + t] = ll[t]; }
    }
  }
}

// Feature values val(0..n-1) at columns [col, col+n), as put8.
template <typename Fn>
__device__ __forceinline__ void put_run(__half* frow, int F, int f32, int col, int n, Fn&& val) {
  for (int k0 = 0; k0 < n; k0 += 8) {
    const int m = min(8, n - k0);
    float v[8];
#pragma unroll
    for (int t = 0; t < 8; ++t) v[t] = t < m ? val(k0 + t) : 0.f;
    put8(frow, F, f32, col + k0, m, v);
  }
}

// 32 feature values from registers at columns [col, col+32), as put8.
__device__ __forceinline__ void put_run32(__half* frow, int F, int f32, int col, const float (&v)[32]) {
#pragma unroll
  for (int k0 = 0; k0 < 32; k0 += 8) {
    float w[8];
#pragma unroll
    for (int t = 0; t < 8; ++t) w[t] = v[k0 + t];
    put8(frow, F, f32, col + k0, 8, w);
  }
}

// Features of residue bi for head h (page "Invariant point attention (IPA)",
// Required behavior): scalar block; local point = R_i^T (sum_j a_ij g_j - t_i),
// its length sqrt(|local|^2 + eps); pair block.  For an empty neighbourhood
// only the (zero) local points are written.  orow = this row's O accumulator divided by l (staged in
// shared memory); (Gx,Gy,Gz) = sum_j a_ij o_G(j), the group-origin part of
// the aggregated value points.  fblk = the (residue, head) block of the
// projection operand, lp = the residue's local points of this head [Q][3].
__device__ void write_features(const CoreArgs& a, size_t bi, bool empty, float* orow, float Gx, float Gy,
                               float Gz, bool with_pair, const float (&R)[9], const float (&t)[3], __half* fblk,
                               float* lp, float* osv) {
  const Plan& p = a.p;
  const int Dv = p.Dv, Q = p.Q, Cz = p.Cz, F = p.Wh8;
  const int sc = 0, xc = Dv, pc = Dv + 4 * Q;
  if (empty) {
    // an empty neighbourhood: the local points are zero; the row's features
    // are not written (the projection selects 0 for the row, whatever they hold)
    if (((3 * Q) & 3) == 0 && (reinterpret_cast<uintptr_t>(lp) & 15) == 0) {
      for (int e = 0; e < 3 * Q; e += 4) *reinterpret_cast<float4*>(lp + e) = make_float4(0.f, 0.f, 0.f, 0.f);
    } else {
      for (int e = 0; e < 3 * Q; ++e) lp[e] = 0.f;
    }
    return;
  }
  auto zero = [](int) { return 0.f; };
  if (p.Wh8 > p.Wh) put_run(fblk, F, p.f32, p.Wh, p.Wh8 - p.Wh, zero);
  // scalar block
  put_run(fblk, F, p.f32, sc, Dv, [&](int d) { return p.f32 ? orow[d] + orow[p.Dv8 + d] : orow[d]; });
  if (osv != nullptr)
    for (int d = 0; d < Dv; ++d) osv[d] = p.f32 ? orow[d] + orow[p.Dv8 + d] : orow[d];
  // points, 8 at a time in registers: aggregate (hi + lo halves + group-origin
  // part), back into the query frame, lengths; then the x, y, z and length
  // feature runs and the local points straight from registers
  const int gofs = p.nsv * p.Dv8;
  const bool lp_vec = (reinterpret_cast<uintptr_t>(lp) & 15) == 0;
  for (int q0 = 0; q0 < Q; q0 += 8) {
    const int nq = min(8, Q - q0);
    float lx[8], ly[8], lz[8], ln[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      lx[u] = ly[u] = lz[u] = ln[u] = 0.f;
      if (u < nq) {
        const int q = q0 + u;
        const float gx = orow[gofs + 3 * q + 0] + orow[gofs + p.Q38 + 3 * q + 0] + Gx - t[0];
        const float gy = orow[gofs + 3 * q + 1] + orow[gofs + p.Q38 + 3 * q + 1] + Gy - t[1];
        const float gz = orow[gofs + 3 * q + 2] + orow[gofs + p.Q38 + 3 * q + 2] + Gz - t[2];
        if (osv != nullptr) {
          osv[Dv + 3 * q + 0] = gx + t[0];
          osv[Dv + 3 * q + 1] = gy + t[1];
          osv[Dv + 3 * q + 2] = gz + t[2];
        }
        lx[u] = R[0] * gx + R[3] * gy + R[6] * gz;
        ly[u] = R[1] * gx + R[4] * gy + R[7] * gz;
        lz[u] = R[2] * gx + R[5] * gy + R[8] * gz;
        ln[u] = sqrtf(lx[u] * lx[u] + ly[u] * ly[u] + lz[u] * lz[u] + a.eps);
      }
    }
    put8(fblk, F, p.f32, xc + q0, nq, lx);
    put8(fblk, F, p.f32, xc + Q + q0, nq, ly);
    put8(fblk, F, p.f32, xc + 2 * Q + q0, nq, lz);
    put8(fblk, F, p.f32, xc + 3 * Q + q0, nq, ln);
    // local points [q][3] of this chunk: 24 floats, 16-byte stores where aligned
    float* lq = lp + 3 * q0;
    if (nq == 8 && lp_vec) {
      float4* l4 = reinterpret_cast<float4*>(lq);
      l4[0] = make_float4(lx[0], ly[0], lz[0], lx[1]);
      l4[1] = make_float4(ly[1], lz[1], lx[2], ly[2]);
      l4[2] = make_float4(lz[2], lx[3], ly[3], lz[3]);
      l4[3] = make_float4(lx[4], ly[4], lz[4], lx[5]);
      l4[4] = make_float4(ly[5], lz[5], lx[6], ly[6]);
      l4[5] = make_float4(lz[6], lx[7], ly[7], lz[7]);
    } else {
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (u < nq) { lq[3 * u] = lx[u]; lq[3 * u + 1] = ly[u]; lq[3 * u + 2] = lz[u]; }
    }
  }
  // pair block through the factors (the tensor-memory path writes it otherwise)
  if (!with_pair) return;
  const int RCz = p.R * Cz;
  if (osv != nullptr)
    for (int rc = 0; rc < RCz; ++rc)
      osv[Dv + 3 * Q + rc] = orow[p.VHp + rc] + (p.f32 ? orow[p.VHp + p.RC8 + rc] : 0.f);
  put_run(fblk, F, p.f32, pc, Cz, [&](int c) {
    float acc = 0.f;
    for (int rr = 0; rr < p.R; ++rr) {
      float u = orow[p.VHp + rr * Cz + c];
      if (p.f32) u += orow[p.VHp + p.RC8 + rr * Cz + c];
      acc = fmaf(ld_any(a.z1, bi * RCz + rr * Cz + c, p.in_f32), u, acc);
    }
    return acc;
  });
}

// Shared-memory use of the feature epilogue, in the Qhat + ring memory:
//   [0]      z1 rows of the query tile [128][R*Cz] (+16 bytes per row), copied
//            during the last key tile, so they sit inside the Qhat buffer
//            (dead once the last QK^T product has completed);
//   [o_off]  O / l of each row, value-head columns [128][staged + 1] fp32.
// z1 is prefetched only where both fit; otherwise the epilogue reads it from
// global memory.
struct EpiLayout {
  bool fast_pair;   // pair block straight from TMEM (Cz a multiple of 32, z1 16-byte aligned)
  bool z1_smem;     // z1 rows prefetched into shared memory
  int staged;       // O columns staged per row
  uint32_t z1_row_bytes, z1_stride, o_off;
};

template <bool SPLIT>
__device__ __forceinline__ EpiLayout epi_layout(const Plan& p, const void* z1) {
  EpiLayout e;
  const uint32_t ring_end = (uint32_t)(p.nQres + (p.vbuf ? p.nVB : 0) + p.nst) * kChunkBytes;
  if (SPLIT && p.oacc_T > 0) {
    // float32 inputs with O in segments: the rows are staged in place in the
    // fp32 accumulator (the tail), all columns, and z1 may use the Qhat region
    e.fast_pair = false;
    e.staged = p.Ocols;
    e.z1_row_bytes = (uint32_t)(p.R * p.Cz * (p.in_f32 ? 4 : 2));
    e.z1_stride = e.z1_row_bytes + 16;
    e.z1_smem = false;
    e.o_off = ring_end + (uint32_t)p.oacc_off;
    return e;
  }
  e.fast_pair = (p.Cz % 32) == 0 && (reinterpret_cast<uintptr_t>(z1) & 15) == 0;
  e.staged = e.fast_pair ? p.VHp : p.Ocols;
  e.z1_row_bytes = (uint32_t)(p.R * p.Cz * (p.in_f32 ? 4 : 2));
  e.z1_stride = e.z1_row_bytes + 16;
  const uint32_t o_bytes = (uint32_t)kTile * (e.staged + 1) * 4;
  e.z1_smem = e.fast_pair && (e.z1_row_bytes & 15) == 0 &&
              (uint32_t)kTile * e.z1_stride <= (uint32_t)p.nQres * kChunkBytes;
  e.o_off = e.z1_smem ? ((uint32_t)kTile * e.z1_stride + 1023u) & ~1023u : 0u;
  if (e.o_off + o_bytes > ring_end) { e.z1_smem = false; e.o_off = 0; }
  return e;
}

// Bounded wait that ignores the abort flag (used only to drain in-flight work).
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity, uint64_t timeout_ns) {
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > timeout_ns) break;
  }
}

// SPLIT: float32 inputs (3-way operands, P as hi + lo, exact point term).
// VB: value-buffer mode (bfloat16 only): each key tile's value chunks [VH | Z]
// land in a buffer of their own and the u lo chunks stream with the keys.
// A query tile without a valid residue (the padding of a short sample): every
// row has an empty neighbourhood, so only the outputs the full path leaves for
// such rows are written (row statistics (-inf, 0), lse -inf, zero local points,
// the row flag and the feature padding) and nothing is computed.  Out of line,
// so the full path's code is unchanged.
__device__ __noinline__ void core_masked_tile(float2* stats, float* lse, uint8_t* rowflag, __half* feat,
                                              float* local_points, int N, int H, int Q, int Kg, int Kgp,
                                              int qt, int h, int b) {
  const int bh = b * H + h;
  for (int r = threadIdx.x; r < kTile; r += blockDim.x) {
    const int i = qt * kTile + r;
    if (i >= N) continue;
    const size_t bi = (size_t)b * N + i;
    stats[(size_t)bh * N + i] = make_float2(-INFINITY, 0.f);
    if (lse != nullptr) lse[(size_t)bh * N + i] = -INFINITY;
    if (h == 0) {
      rowflag[bi] = 0;
      for (int c = Kg; c < Kgp; ++c) feat[bi * Kgp + c] = __float2half_rn(0.f);
    }
    float* lp = local_points + (bi * H + h) * (size_t)Q * 3;
    for (int e = 0; e < 3 * Q; ++e) lp[e] = 0.f;
  }
}

// SAVE: also store the normalised aggregates of every row (training recompute).
template <bool SPLIT, bool VB, bool SAVE>
__global__ void __launch_bounds__(256, 1)
fipa_core_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmKH,
                 const __grid_constant__ CUtensorMap tmVH, const __grid_constant__ CUtensorMap tmZ,
                 const CoreArgs a) {
  {
    const int qt0 = blockIdx.x + a.p.row0 / kTile;
    if (a.flag[(size_t)blockIdx.z * a.p.nT + qt0] == 0) {   // uniform over the CTA
      core_masked_tile(a.stats, a.lse, a.rowflag, a.feat, a.local_points, a.p.N, a.p.H, a.p.Q, a.p.Kg, a.p.Kgp,
                       qt0, blockIdx.y, blockIdx.z);
      return;
    }
  }
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const Plan& p = a.p;
  // CTA timeline (debug trace only): the last 8 slots of the softmax role's log
  const bool timeline = a.trace != nullptr && threadIdx.x == 128 &&
                        (int)(blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z)) == a.trace_cta;
  Tracer ttr{timeline ? a.trace + (size_t)2 * 2 * kTraceCap : nullptr, kTraceCap - 8};
  ttr.ev(40);
  uint8_t* sQ = smem;                                        // resident Qhat chunks
  uint8_t* sV = sQ + p.nQres * kChunkBytes;                  // value buffer (value-buffer mode)
  uint8_t* sRing = sV + (VB ? p.nVB : 0) * kChunkBytes;
  uint8_t* tail = sRing + p.nst * kChunkBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(tail + kBarFull);
  uint64_t* empty = reinterpret_cast<uint64_t*>(tail + kBarEmpty);
  uint64_t* q_full = reinterpret_cast<uint64_t*>(tail + kBarQ);
  uint64_t* s_full = reinterpret_cast<uint64_t*>(tail + kBarSFull);
  uint64_t* s_free = reinterpret_cast<uint64_t*>(tail + kBarSFree);
  uint64_t* p_full = reinterpret_cast<uint64_t*>(tail + kBarPFull);
  uint64_t* pv_done = reinterpret_cast<uint64_t*>(tail + kBarPVDone);
  uint64_t* kt_full = reinterpret_cast<uint64_t*>(tail + kBarKtFull);
  uint64_t* kt_empty = reinterpret_cast<uint64_t*>(tail + kBarKtEmpty);
  uint64_t* drain = reinterpret_cast<uint64_t*>(tail + kBarDrain);
  uint64_t* v_full = reinterpret_cast<uint64_t*>(tail + kBarVFull);
  float* ktbuf = reinterpret_cast<float*>(tail + kKtBuf);
  float4* okbuf = reinterpret_cast<float4*>(tail + kOkBuf);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tail + kMisc);
  int* abort_flag = reinterpret_cast<int*>(tail + kMisc + 4);
  int* ntiles = reinterpret_cast<int*>(tail + kMisc + 8);
  uint16_t* tiles = reinterpret_cast<uint16_t*>(tail + kTiles);
  float* kpbuf = reinterpret_cast<float*>(tail + kKpBuf);          // [2][128][3P] (SPLIT only)

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = blockIdx.x + p.row0 / kTile, h = blockIdx.y, b = blockIdx.z;
  const int bh = b * p.H + h;
  const int N = p.N, nT = p.nT;

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.nst; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    mbar_init(q_full, 1);
    mbar_init(s_full, 1);
    mbar_init(s_free, 128);
    mbar_init(p_full, 128);
    mbar_init(pv_done, 1);
    mbar_init(&kt_full[0], 64);
    mbar_init(&kt_full[1], 64);
    mbar_init(&kt_empty[0], 128);
    mbar_init(&kt_empty[1], 128);
    mbar_init(drain, 1);
    mbar_init(v_full, 1);
    fence_mbar_init();
    *abort_flag = 0;
    // key tiles with a valid residue: the query's own tile first (it usually
    // holds the row maximum, so the running max rarely needs a rescale)
    int n = 0;
    const int* fl = a.flag + (size_t)b * nT;
    if (fl[qt]) {
      tiles[n++] = (uint16_t)qt;
      for (int t = 0; t < nT; ++t)
        if (t != qt && fl[t]) tiles[n++] = (uint16_t)t;
    }
    *ntiles = n;
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int nkt = *ntiles;
  const WaitCtx wc{abort_flag, a.status, a.timeout_ns};
  ttr.ev(41);
  const int lin_cta = blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z);
  long long* tbase = (a.trace != nullptr && lin_cta == a.trace_cta) ? a.trace : nullptr;
  auto tracer = [&](int role) { return Tracer{tbase ? tbase + (size_t)role * 2 * kTraceCap : nullptr, 0}; };
  // per-row softmax state, read by the fused feature epilogue after the roles end
  float rowM = -INFINITY, rowL = 0.f, rowW[3] = {0.f, 0.f, 0.f};
  bool row_ok = false;
  float rowR[9], rowT[3];   // frame of the row's residue, loaded during the last tile

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && nkt > 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmKH);
      tma_prefetch_desc(&tmVH);
      tma_prefetch_desc(&tmZ);
      mbar_arrive_expect_tx(q_full, (uint32_t)(p.nQres * kChunkBytes));
      for (int c = 0; c < p.nQres; ++c) tma_load_3d(sQ + c * kChunkBytes, &tmQ, q_full, c * kChunk, qt * kTile, bh);
      int st = 0;
      uint32_t ph = 0;
      bool ok = true;
      uint32_t issued = 0;
      Tracer tr = tracer(0);
      auto push = [&](const CUtensorMap* tm, int c0, int c1, int c2) {
        if (!ok) return;
        tr.ev(1);
        if (!mbar_wait(&empty[st], ph ^ 1u, wc, 1)) { ok = false; return; }
        mbar_arrive_expect_tx(&full[st], kChunkBytes);
        tma_load_3d(sRing + st * kChunkBytes, tm, &full[st], c0, c1, c2);
        tr.ev(2);
        ++issued;
        if (++st == p.nst) { st = 0; ph ^= 1u; }
      };
      auto push_qk = [&](int kt) {
        for (int c = 0; c < p.nZ; ++c) {
          push(&tmZ, c * kChunk, kt * kTile, b);
          // value-buffer mode: the u lo chunk that meets this z2 chunk
          if (VB) push(&tmQ, (p.nKH + p.nZ + c) * kChunk, qt * kTile, bh);
        }
        for (int c = 0; c < p.nKH; ++c) push(&tmKH, c * kChunk, kt * kTile, bh);
      };
      auto push_pv = [&](int kt) {
        for (int c = 0; c < p.nVH; ++c) push(&tmVH, c * kChunk, kt * kTile, bh);
        for (int c = 0; c < p.nZV; ++c) push(&tmZ, c * kChunk, kt * kTile, b);
      };
      push_qk(tiles[0]);
      for (int s = 0; s < nkt && ok; ++s) {
        if (s + 1 < nkt) push_qk(tiles[s + 1]);
        if (!VB) push_pv(tiles[s]);   // value-buffer mode: the MMA thread loads them
      }
      if (*abort_flag) {
        // wind down: let every load already issued land before the CTA exits
        drain_wait(q_full, 0, a.timeout_ns);
        const uint32_t last = issued < (uint32_t)p.nst ? issued : (uint32_t)p.nst;
        for (uint32_t k = 0; k < last; ++k) {
          const uint32_t n = issued - 1 - k;              // push index
          drain_wait(&full[n % p.nst], (n / p.nst) & 1u, a.timeout_ns);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && nkt > 0) {
      Tracer tr = tracer(1);
      bool ok = mbar_wait(q_full, 0, wc, 2);
      tr.ev(10);
      tc_fence_after();
      int st = 0;
      uint32_t ph = 0;
      const uint32_t idS = idesc_f16(128, 128, 0, 0);
      const uint32_t sQa = smem_u32(sQ), sRa = smem_u32(sRing);
      // value-buffer mode: the value chunks of key tile `kt` go to their own
      // buffer; issued only once the P.V product that read it before is done
      uint32_t v_issued = 0;
      auto load_v = [&](int kt) {
        mbar_arrive_expect_tx(v_full, (uint32_t)(p.nVB * kChunkBytes));
        for (int c = 0; c < p.nVH; ++c) tma_load_3d(sV + c * kChunkBytes, &tmVH, v_full, c * kChunk, kt * kTile, bh);
        for (int c = 0; c < p.nZV; ++c)
          tma_load_3d(sV + (p.nVH + c) * kChunkBytes, &tmZ, v_full, c * kChunk, kt * kTile, b);
        ++v_issued;
      };
      int v_pend = -1;                      // key-tile index s whose values wait for P.V(s-1)
      auto poll_v = [&](bool block) -> bool {
        if (v_pend < 0) return true;
        const uint32_t par = (uint32_t)(v_pend - 1) & 1u;
        if (block) {
          if (!mbar_wait(pv_done, par, wc, 12)) return false;
        } else if (!mbar_try_wait(pv_done, par)) {
          return true;
        }
        load_v(tiles[v_pend]);
        v_pend = -1;
        return true;
      };
      // P.V(s) over the value buffer as a flat sequence of K-steps: runs of up
      // to 4 64-column groups (N = 64 x run, groups 16 KB apart), 8 K-steps of
      // 16 keys each.  (Issuing it in pieces between the QK^T(s+1) chunks was
      // measured slower: the logits of the next tile then wait for it.)
      auto mma_qk_vbuf = [&]() -> bool {
        // ring order: per z2 chunk, [z2 | u lo]; the z2 chunk meets the resident
        // u hi chunk and the streamed u lo chunk; then the head part.  The small
        // pair terms accumulate before the large point terms.
        for (int c = 0; c < p.nZ; ++c) {
          tr.ev(11);
          if (!mbar_wait(&full[st], ph, wc, 3)) return false;
          tr.ev(12);
          const int sz = st;
          if (++st == p.nst) { st = 0; ph ^= 1u; }
          tc_fence_after();
          const uint32_t b0 = sRa + sz * kChunkBytes;
          const uint32_t ah = sQa + (p.nKH + c) * kChunkBytes;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ss(tmem + kTmemS, desc_kmajor_sw128(ah + kk * 32), desc_kmajor_sw128(b0 + kk * 32), idS,
                   (c | kk) != 0 ? 1u : 0u);
          // the u lo half, as soon as its chunk has landed
          tr.ev(11);
          if (!mbar_wait(&full[st], ph, wc, 3)) return false;
          tr.ev(12);
          const int sl = st;
          if (++st == p.nst) { st = 0; ph ^= 1u; }
          tc_fence_after();
          const uint32_t al = sRa + sl * kChunkBytes;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ss(tmem + kTmemS, desc_kmajor_sw128(al + kk * 32), desc_kmajor_sw128(b0 + kk * 32), idS, 1u);
          tc_commit(&empty[sz]);
          tc_commit(&empty[sl]);
          if (!poll_v(false)) return false;
        }
        for (int c = 0; c < p.nKH; ++c) {
          tr.ev(11);
          if (!mbar_wait(&full[st], ph, wc, 3)) return false;
          tr.ev(12);
          tc_fence_after();
          const uint32_t b0 = sRa + st * kChunkBytes, a0 = sQa + c * kChunkBytes;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ss(tmem + kTmemS, desc_kmajor_sw128(a0 + kk * 32), desc_kmajor_sw128(b0 + kk * 32), idS, 1u);
          tc_commit(&empty[st]);
          if (++st == p.nst) { st = 0; ph ^= 1u; }
        }
        tc_commit(s_full);
        tr.ev(17);
        return true;
      };
      auto mma_pv_vbuf = [&](int s) -> bool {
        if (!mbar_wait(v_full, (uint32_t)s & 1u, wc, 13)) return false;
        tc_fence_after();
        const uint32_t v0 = smem_u32(sV);
        for (int c = 0; c < p.nVB; c += 4) {
          const int run = p.nVB - c < 4 ? p.nVB - c : 4;
          const uint32_t b0 = v0 + c * kChunkBytes;
          const uint32_t idO = idesc_f16(128, 64 * run, 0, 1);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ts(tmem + (uint32_t)(p.tmemO + c * kChunk), tmem + kTmemP + kk * 8,
                   desc_mnmajor_sw128(b0 + kk * 2048, kChunkBytes), idO, (s > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(pv_done);
        tr.ev(18);
        return true;
      };
      auto mma_qk = [&]() -> bool {
        if (VB) return mma_qk_vbuf();
        // key chunks in ring order: the pair part first (each z2 chunk meets nqz
        // Qhat chunks: u hi, u lo), the head part (scalar and point columns)
        // last, so the small pair terms accumulate before the large point terms
        const int nb = p.nZ + p.nKH;
        for (int c = 0; c < nb; ++c) {
          tr.ev(11);
          if (!mbar_wait(&full[st], ph, wc, 3)) return false;
          tr.ev(12);
          tc_fence_after();
          const uint32_t b0 = sRa + st * kChunkBytes;
          const bool pair = c < p.nZ;
          const int na = pair ? p.nqz : 1;
          for (int qz = 0; qz < na; ++qz) {
            const int ac = pair ? p.nKH + qz * p.nZ + c : c - p.nZ;
            const uint32_t a0 = sQa + ac * kChunkBytes;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_ss(tmem + kTmemS, desc_kmajor_sw128(a0 + kk * 32), desc_kmajor_sw128(b0 + kk * 32), idS,
                     (c | qz | kk) != 0 ? 1u : 0u);
          }
          tc_commit(&empty[st]);
          if (++st == p.nst) { st = 0; ph ^= 1u; }
        }
        tc_commit(s_full);
        tr.ev(17);
        return true;
      };
      auto mma_pv = [&](int s) -> bool {
        if (VB) return mma_pv_vbuf(s);
        // value chunks in O-column order; up to 4 chunks in consecutive ring
        // slots form one MMA of N = 64 x run (MN-major B, groups 16 KB apart)
        const int nchunk = p.nVH + p.nZV;
        for (int c = 0; c < nchunk;) {
          int run = nchunk - c;
          if (run > 4) run = 4;
          if (run > p.nst - st) run = p.nst - st;
          for (int u = 0; u < run; ++u) {
            tr.ev(11);
            if (!mbar_wait(&full[st + u], ph, wc, 4)) return false;
            tr.ev(12);
          }
          tc_fence_after();
          const uint32_t b0 = sRa + st * kChunkBytes;
          const uint32_t dcol = tmem + (uint32_t)(p.tmemO + c * kChunk);
          const uint32_t idO = idesc_f16(128, 64 * run, 0, 1);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t bd = desc_mnmajor_sw128(b0 + kk * 2048, kChunkBytes);
            uint32_t acc0 = (s > 0 || kk > 0) ? 1u : 0u;
            if (SPLIT && p.oacc_T > 0) acc0 = (s % p.oacc_T != 0 || kk > 0) ? 1u : 0u;
            mma_ts(dcol, tmem + kTmemP + kk * 8, bd, idO, acc0);
            if (SPLIT) mma_ts(dcol, tmem + kTmemP + 64 + kk * 8, bd, idO, 1u);
          }
          for (int u = 0; u < run; ++u) tc_commit(&empty[st + u]);
          st += run;
          if (st == p.nst) { st = 0; ph ^= 1u; }
          c += run;
        }
        tc_commit(pv_done);
        tr.ev(18);
        return true;
      };
      if (ok && VB) load_v(tiles[0]);
      if (ok) ok = mma_qk();
      for (int s = 0; ok && s < nkt; ++s) {
        if (s + 1 < nkt) {
          tr.ev(13);
          if (!mbar_wait(s_free, s & 1, wc, 5)) break;
          tr.ev(14);
          tc_fence_after();
          if (!mma_qk()) break;
        }
        if (VB && !poll_v(true)) break;   // this tile's values, if QK^T did not load them yet
        tr.ev(15);
        if (!mbar_wait(p_full, s & 1, wc, 6)) break;
        tr.ev(16);
        tc_fence_after();
        if (!mma_pv(s)) break;
        if (VB && s + 1 < nkt) v_pend = s + 1;   // loads once P.V(s) has read the buffer
      }
      // every MMA this thread issued has finished, and the last value load has
      // landed, before the CTA tears down
      tc_commit(drain);
      drain_wait(drain, 0, a.timeout_ns);
      if (v_issued > 0) drain_wait(v_full, (v_issued - 1) & 1u, a.timeout_ns);
    }
  } else if (warp == 2 || warp == 3) {
    // ------------------------------------------------------------ per-key terms
    // kterm[s][j] = -g sum_p |b'_p|^2 + 2g D_sj . sum_p b'_p  (-inf for a masked or
    // absent key), D_sj = origin of query group s - origin of key j's group; the
    // four key-group origins of the tile go to shared memory as well.
    const int tt = threadIdx.x - 64;
    Tracer ktr = tracer(3);
    const float g = point_weight(load_raw(a, h), p.P);
    float4 oq[4];
#pragma unroll
    for (int sq = 0; sq < 4; ++sq) oq[sq] = a.orig[(size_t)b * p.nG + qt * 4 + sq];
    for (int s = 0; s < nkt; ++s) {
      const int kb = s & 1;
      const bool okw = mbar_wait(&kt_empty[kb], ((s >> 1) & 1) ^ 1, wc, 10);
      if (!__all_sync(0xffffffffu, okw)) break;
      if (tt == 0) ktr.ev(30);
      const int kt = tiles[s];
      if (tt < 4) okbuf[kb * 4 + tt] = a.orig[(size_t)b * p.nG + kt * 4 + tt];
      for (int e = tt; e < kTile; e += 64) {
        const int j = kt * kTile + e;
        const float4 ok = a.orig[(size_t)b * p.nG + kt * 4 + (e >> 5)];
        float4 kv = make_float4(-INFINITY, 0.f, 0.f, 0.f);
        if (j < N) kv = a.kvec[(size_t)bh * N + j];
#pragma unroll
        for (int sq = 0; sq < 4; ++sq) {
          const float dx = oq[sq].x - ok.x, dy = oq[sq].y - ok.y, dz = oq[sq].z - ok.z;
          ktbuf[(kb * 4 + sq) * kTile + e] = SPLIT ? kv.x : kv.x + 2.f * g * (dx * kv.y + dy * kv.z + dz * kv.w);
        }
      }
      if (SPLIT) {
        // float32 inputs: the key tile's points b' for the exact fp32 distance
        const int P3 = 3 * p.P;
        float* kpb = kpbuf + kb * kTile * P3;
        const size_t base = ((size_t)bh * N + (size_t)kt * kTile) * P3;
        const size_t lim = (size_t)(N - kt * kTile) * P3;
        for (int e = tt; e < kTile * P3; e += 64) kpb[e] = (size_t)e < lim ? a.KP[base + e] : 0.f;
      }
      mbar_arrive(&kt_full[kb]);
      if (tt == 0) ktr.ev(31);
    }
  } else {
    // ------------------------------------------------------------ softmax warps
    // One thread per query row; the warp's TMEM lane quadrant is also the row's
    // 32-residue origin group.  Per key tile and 32-key group t the row term is
    // rc_t = -g (P |D_t|^2 + 2 D_t . sum_p a'_p); it rides in the exp's FMA addend.
    const int wq = warp - 4;
    const int r = wq * 32 + lane;
    const int i = qt * kTile + r;
    const bool in_range = i < N;
    const bool row_valid = in_range && a.mask[(size_t)b * N + i] != 0;
    const float4 qv = in_range ? a.qvec[(size_t)bh * N + i] : make_float4(0.f, 0.f, 0.f, 0.f);
    const float4 oqs = a.orig[(size_t)b * p.nG + qt * 4 + wq];
    const float g = point_weight(load_raw(a, h), p.P);
    const uint32_t trow = tmem + ((uint32_t)(wq * 32) << 16);
    const uint8_t* pmrow = (a.pair_mask != nullptr && in_range) ? a.pair_mask + ((size_t)b * N + i) * N : nullptr;
    float M = -INFINITY, l = 0.f, Wx = 0.f, Wy = 0.f, Wz = 0.f;
    bool ok = true;
    Tracer str = tracer(2);
    if (threadIdx.x != 128) str.buf = nullptr;
    // float32 inputs: this row's fp32 accumulator of the flushed O segments
    const bool oseg = SPLIT && p.oacc_T > 0;
    float* accrow = oseg ? reinterpret_cast<float*>(tail + p.oacc_off) + (size_t)(wq * 32 + lane) * (p.Ocols + 1)
                         : nullptr;
    if (oseg)
      for (int c = 0; c <= p.Ocols; ++c) accrow[c] = 0.f;
    for (int s = 0; s < nkt; ++s) {
      const int kt = tiles[s];
      const int kb = s & 1;

      str.ev(20);
      ok = mbar_wait(s_full, s & 1, wc, 7);
      str.ev(21);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      tc_fence_after();
      uint32_t sv[4][32];
      tmem_ld32(trow + kTmemS + 0, sv[0]);
      tmem_ld32(trow + kTmemS + 32, sv[1]);
      tmem_ld32(trow + kTmemS + 64, sv[2]);
      tmem_ld32(trow + kTmemS + 96, sv[3]);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(s_free);
      str.ev(22);

      ok = mbar_wait(&kt_full[kb], (s >> 1) & 1, wc, 11);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      str.ev(23);
      float4 okg[4];
      float rc[4];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        okg[t] = okbuf[kb * 4 + t];
        const float dx = oqs.x - okg[t].x, dy = oqs.y - okg[t].y, dz = oqs.z - okg[t].z;
        rc[t] = SPLIT ? 0.f
                      : -g * ((float)p.P * (dx * dx + dy * dy + dz * dz) + 2.f * (dx * qv.x + dy * qv.y + dz * qv.z));
      }
      const float4* kb4 = reinterpret_cast<const float4*>(ktbuf + (kb * 4 + wq) * kTile);
#pragma unroll
      for (int t = 0; t < 4; ++t) {
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          const float4 kt4 = kb4[(t * 32 + e) >> 2];
          sv[t][e + 0] = __float_as_uint(__uint_as_float(sv[t][e + 0]) + kt4.x);
          sv[t][e + 1] = __float_as_uint(__uint_as_float(sv[t][e + 1]) + kt4.y);
          sv[t][e + 2] = __float_as_uint(__uint_as_float(sv[t][e + 2]) + kt4.z);
          sv[t][e + 3] = __float_as_uint(__uint_as_float(sv[t][e + 3]) + kt4.w);
        }
      }
      if (SPLIT) {
        // float32 inputs: -g sum_p |a'_p + D_t - b'_p|^2 taken directly in fp32
        const int P3 = 3 * p.P;
        const float* kpb = kpbuf + kb * kTile * P3;
        float aq[3 * kMaxPSimt];
        for (int x = 0; x < P3; ++x) aq[x] = in_range ? a.QP[((size_t)bh * N + i) * P3 + x] : 0.f;
        // per group of 32 keys: one pass over the coordinates with 32 accumulators
        // in registers (each key's sum still runs over x in order); a pass per
        // key instead indexed aq and dd at run time, i.e. from local memory,
        // and made this loop the float32 core's bound (3.6x slower at N = 4096)
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const float dd[3] = {oqs.x - okg[t].x, oqs.y - okg[t].y, oqs.z - okg[t].z};
          float d2[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) d2[e] = 0.f;
          const float* kt0 = kpb + t * 32 * P3;
          if ((P3 & 3) == 0) {
            // four coordinates of a key per 16-byte load (rows of 3P floats stay
            // 16-byte aligned), added in the same order
            for (int x = 0; x < P3; x += 4) {
              float ax[4];
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                const int c = (x + u) % 3;
                ax[u] = aq[x + u] + (c == 0 ? dd[0] : (c == 1 ? dd[1] : dd[2]));
              }
#pragma unroll
              for (int e = 0; e < 32; ++e) {
                const float4 kv = *reinterpret_cast<const float4*>(kt0 + e * P3 + x);
                float d = ax[0] - kv.x;
                d2[e] = fmaf(d, d, d2[e]);
                d = ax[1] - kv.y;
                d2[e] = fmaf(d, d, d2[e]);
                d = ax[2] - kv.z;
                d2[e] = fmaf(d, d, d2[e]);
                d = ax[3] - kv.w;
                d2[e] = fmaf(d, d, d2[e]);
              }
            }
          } else {
            for (int x = 0; x < P3; ++x) {
              const int c = x % 3;
              const float ax = aq[x] + (c == 0 ? dd[0] : (c == 1 ? dd[1] : dd[2]));
#pragma unroll
              for (int e = 0; e < 32; ++e) {
                const float d = ax - kt0[e * P3 + x];
                d2[e] = fmaf(d, d, d2[e]);
              }
            }
          }
#pragma unroll
          for (int e = 0; e < 32; ++e) sv[t][e] = __float_as_uint(__uint_as_float(sv[t][e]) - g * d2[e]);
        }
      }
      mbar_arrive(&kt_empty[kb]);
      if (pmrow != nullptr) {
#pragma unroll
        for (int t = 0; t < 4; ++t) {
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const int j = kt * kTile + t * 32 + e;
            if (j >= N || pmrow[j] == 0) sv[t][e] = __float_as_uint(-INFINITY);
          }
        }
      }
      // tile maximum of the true logits (log2 units, minus -g sum|a'|^2)
      float mtile = -INFINITY;
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        float mx = -INFINITY;
#pragma unroll
        for (int e = 0; e < 32; ++e) mx = fmaxf(mx, __uint_as_float(sv[t][e]));
        mtile = fmaxf(mtile, (mx + rc[t]) * kLog2e);
      }
      if (!row_valid) mtile = -INFINITY;

      // lazily updated running max: rescale only when it grows by more than 2^kTau
      float alpha = 1.f;
      bool resc = false;
      if (mtile > M + kTau) {
        resc = (M != -INFINITY);
        alpha = resc ? ex2_approx(M - mtile) : 0.f;
        M = mtile;
        l *= alpha; Wx *= alpha; Wy *= alpha; Wz *= alpha;
      }

      uint32_t pk[2][32];
      uint32_t plo[2][32];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const float mb = row_valid ? (M == -INFINITY ? 0.f : M - rc[t] * kLog2e) : INFINITY;
        float rs0 = 0.f, rs1 = 0.f;
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          const float p0 = ex2_approx(fmaf(__uint_as_float(sv[t][e + 0]), kLog2e, -mb));
          const float p1 = ex2_approx(fmaf(__uint_as_float(sv[t][e + 1]), kLog2e, -mb));
          const float p2 = ex2_approx(fmaf(__uint_as_float(sv[t][e + 2]), kLog2e, -mb));
          const float p3 = ex2_approx(fmaf(__uint_as_float(sv[t][e + 3]), kLog2e, -mb));
          const int w = (t & 1) * 16 + e / 2;
          pk[t >> 1][w] = pack_half2(p0, p1);
          pk[t >> 1][w + 1] = pack_half2(p2, p3);
          if (!SPLIT) {
            // normalise with the sum of the fp16 weights the P.V product uses
            const float2 f01 = __half22float2(*reinterpret_cast<const __half2*>(&pk[t >> 1][w]));
            const float2 f23 = __half22float2(*reinterpret_cast<const __half2*>(&pk[t >> 1][w + 1]));
            rs0 += f01.x + f01.y;
            rs1 += f23.x + f23.y;
          } else {
            rs0 += p0 + p1;
            rs1 += p2 + p3;
          }
          if (SPLIT) {
            const __half2 h01 = *reinterpret_cast<const __half2*>(&pk[t >> 1][w]);
            const __half2 h23 = *reinterpret_cast<const __half2*>(&pk[t >> 1][w + 1]);
            plo[t >> 1][w] = pack_half2(p0 - __low2float(h01), p1 - __high2float(h01));
            plo[t >> 1][w + 1] = pack_half2(p2 - __low2float(h23), p3 - __high2float(h23));
          }
        }
        const float rs = rs0 + rs1;
        l += rs;
        Wx += okg[t].x * rs; Wy += okg[t].y * rs; Wz += okg[t].z * rs;
      }

      // P and O are free once the previous P.V product has finished
      str.ev(24);
      if (s > 0) {
        ok = mbar_wait(pv_done, (s - 1) & 1, wc, 8);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        tc_fence_after();
      }
      str.ev(25);
      if (oseg && s > 0 && s % p.oacc_T == 0) {
        // close the tensor-memory segment: O joins the row's accumulator (both
        // rescaled to the current maximum) and P.V(s) starts a fresh one
        const float f = resc ? alpha : 1.f;
        for (int c = 0; c < p.Ocols; c += 32) {
          uint32_t o[32];
          tmem_ld32(trow + (uint32_t)(p.tmemO + c), o);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) accrow[c + e] = (accrow[c + e] + __uint_as_float(o[e])) * f;
        }
      } else if (__any_sync(0xffffffffu, resc)) {
        const float f = resc ? alpha : 1.f;
        for (int c = 0; c < p.Ocols; c += 32) {
          uint32_t o[32];
          tmem_ld32(trow + (uint32_t)(p.tmemO + c), o);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * f);
          tmem_st32(trow + (uint32_t)(p.tmemO + c), o);
        }
        if (oseg)
          for (int c = 0; c < p.Ocols; ++c) accrow[c] *= f;
      }
      tmem_st32(trow + kTmemP, pk[0]);
      tmem_st32(trow + kTmemP + 32, pk[1]);
      if (SPLIT) {
        tmem_st32(trow + kTmemP + 64, plo[0]);
        tmem_st32(trow + kTmemP + 96, plo[1]);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(p_full);
      str.ev(26);
    }
    {
      // every QK^T product has completed (the last logits were read), so the
      // Qhat buffer is free: prefetch this row's z1 factors and frame while the
      // last P.V product runs
      const int i = qt * kTile + wq * 32 + lane;
      const size_t bi = (size_t)b * N + (i < N ? i : 0);
#pragma unroll
      for (int e = 0; e < 9; ++e) rowR[e] = ld_any(a.rot, bi * 9 + e, p.in_f32);
#pragma unroll
      for (int e = 0; e < 3; ++e) rowT[e] = ld_any(a.trans, bi * 3 + e, p.in_f32);
      const EpiLayout el = epi_layout<SPLIT>(p, a.z1);
      if (el.z1_smem && i < N) {
        const uint8_t* src = static_cast<const uint8_t*>(a.z1) + bi * el.z1_row_bytes;
        uint8_t* dst = smem + (size_t)(wq * 32 + lane) * el.z1_stride;
        for (uint32_t o = 0; o < el.z1_row_bytes; o += 16) cp_async16(dst + o, src + o);
      }
      cp_async_commit();
    }
    if (ok && nkt > 0) {
      ok = mbar_wait(pv_done, (nkt - 1) & 1, wc, 9);
      ok = __all_sync(0xffffffffu, ok);
      tc_fence_after();
    }
    rowM = M; rowL = l; rowW[0] = Wx; rowW[1] = Wy; rowW[2] = Wz;
    row_ok = ok;
  }

  // ------------------------------------------------- fused feature epilogue
  // Every MMA has finished and every TMA load has landed, so the Qhat and ring
  // shared memory is reused to stage each row's value-head accumulators (row
  // stride +1 float: conflict-free).  Each softmax thread then builds the
  // features of its (residue, head): the page's scalar block, the aggregated
  // global points taken back into the query frame, their lengths, and the pair
  // block through the factors, sum_r z1[i,r,c] U[r,c].
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  ttr.ev(42);
  const EpiLayout el = epi_layout<SPLIT>(p, a.z1);
  const bool fast_pair = el.fast_pair;
  // per-row state for the warps that did not run the softmax (the key-term
  // buffer is free now); the z1 copies of the softmax threads complete first
  float2* rowinfo = reinterpret_cast<float2*>(tail + kKtBuf);
  // float32 inputs: the P.V product's own sum of P (the value column of ones),
  // which normalises O: the tensor cores' fp32 accumulation of the aggregates
  // then shares its rounding with the divisor, instead of drifting from the
  // softmax's CUDA-core sum as the number of keys grows
  float* rowlsum = reinterpret_cast<float*>(tail + kKtBuf + kTile * 8);
  if (warp >= 4) {
    cp_async_wait_all();
    rowinfo[(warp - 4) * 32 + lane] = make_float2(rowL, (row_ok && nkt > 0) ? 1.f : 0.f);
    if (SPLIT && p.ones_col >= 0) {
      float lt = 0.f;
      const bool aborted = __any_sync(0xffffffffu, *abort_flag != 0);
      if (nkt > 0 && !aborted) {                               // uniform over the warp
        uint32_t o[32];
        tmem_ld32(tmem + ((uint32_t)((warp - 4) * 32) << 16) + (uint32_t)(p.tmemO + (p.ones_col & ~31)), o);
        tmem_ld_wait();
        lt = __uint_as_float(o[p.ones_col & 31]);
        if (p.oacc_T > 0)
          lt += reinterpret_cast<float*>(tail + p.oacc_off)[(size_t)((warp - 4) * 32 + lane) * (p.Ocols + 1) + p.ones_col];
      }
      rowlsum[(warp - 4) * 32 + lane] = lt;
    }
  }
  __syncthreads();
  if (*abort_flag == 0) {
    // warps w and w+4 serve the same 32 rows (TMEM lane quadrant w % 4):
    // warps 4-7 the scalar, point and length features, warps 0-3 the pair block
    const int wq = warp & 3;
    const int r = wq * 32 + lane;
    const int i = qt * kTile + r;
    const bool in_range = i < N;
    const uint32_t trow = tmem + ((uint32_t)(wq * 32) << 16);
    const float2 ri = rowinfo[r];
    const float inv = ri.x > 0.f ? 1.f / ri.x : 0.f;
    float inv_o = inv;                                        // divisor of the P.V aggregates
    if (SPLIT && p.ones_col >= 0) {
      const float lt = rowlsum[r];
      inv_o = lt > 0.f ? 1.f / lt : inv;
    }
    const bool live = ri.y != 0.f;
    const bool empty = !(ri.x > 0.f) || !live;
    const size_t bi = (size_t)b * N + (in_range ? i : 0);
    // this row's head block of the projection operand and its local points
    __half* fblk = a.feat + bi * p.Kgp + (size_t)h * p.nseg * p.Wh8;
    if (warp >= 4) {
      const int staged = el.staged;                         // columns staged in shared memory
      float* orow = reinterpret_cast<float*>(smem + el.o_off) + (size_t)r * (staged + 1);
      if (live) {
        for (int c = 0; c < staged; c += 32) {
          uint32_t o[32];
          tmem_ld32(trow + (uint32_t)(p.tmemO + c), o);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e)
            orow[c + e] = (SPLIT && p.oacc_T > 0 ? orow[c + e] + __uint_as_float(o[e]) : __uint_as_float(o[e])) * inv_o;
        }
      }
      ttr.ev(45);
      float* lp = a.local_points + (bi * p.H + h) * (size_t)p.Q * 3;
      if (in_range) {
        a.stats[(size_t)bh * N + i] = make_float2(rowM, rowL);
        if (a.lse != nullptr) {
          const float4 qv = a.qvec[(size_t)bh * N + i];
          a.lse[(size_t)bh * N + i] = rowL > 0.f ? (rowM + log2f(rowL)) * kLn2 + qv.w : -INFINITY;
        }
        if (h == 0) a.rowflag[bi] = empty ? 0 : 1;
        if (h == 0)
          for (int c = p.Kg; c < p.Kgp; ++c) a.feat[bi * p.Kgp + c] = __float2half_rn(0.f);
        float* osv = SAVE ? a.osave + (bi * p.H + h) * (size_t)(p.Dv + 3 * p.Q + p.R * p.Cz) : nullptr;
        write_features(a, bi, empty, orow, rowW[0] * inv, rowW[1] * inv, rowW[2] * inv, !fast_pair, rowR, rowT,
                       fblk, lp, osv);
      }
      ttr.ev(46);
    } else if (fast_pair) {
      // pair block straight from tensor memory, 32 channels at a time
      const int Cz = p.Cz, RCz = p.R * Cz, pcol = p.Dv + 4 * p.Q;
      __half* frow = fblk;
      const uint8_t* zs = smem + (size_t)r * el.z1_stride;
      for (int c0 = 0; c0 < Cz; c0 += 32) {
        float acc[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) acc[e] = 0.f;
        for (int rr = 0; rr < p.R; ++rr) {
          uint32_t o[32];
          if (live) {
            tmem_ld32(trow + (uint32_t)(p.tmemO + p.VHp + rr * Cz + c0), o);
            tmem_ld_wait();
            if (p.f32) {
              uint32_t o2[32];
              tmem_ld32(trow + (uint32_t)(p.tmemO + p.VHp + p.RC8 + rr * Cz + c0), o2);
              tmem_ld_wait();
#pragma unroll
              for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) + __uint_as_float(o2[e]));
            }
          }
          if (in_range && !empty) {
            const size_t zoff = bi * RCz + (size_t)rr * Cz + c0;
            const size_t zrel = (size_t)rr * Cz + c0;
            float zv[32];
            if (p.in_f32) {
              const float4* z4 = el.z1_smem ? reinterpret_cast<const float4*>(zs) + zrel / 4
                                         : reinterpret_cast<const float4*>(static_cast<const float*>(a.z1) + zoff);
#pragma unroll
              for (int k = 0; k < 8; ++k) {
                const float4 t4 = el.z1_smem ? z4[k] : __ldg(z4 + k);
                zv[4 * k] = t4.x; zv[4 * k + 1] = t4.y; zv[4 * k + 2] = t4.z; zv[4 * k + 3] = t4.w;
              }
            } else {
              const uint4* z4 = el.z1_smem ? reinterpret_cast<const uint4*>(zs) + zrel / 8
                                        : reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.z1) + zoff);
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                const uint4 t4 = el.z1_smem ? z4[k] : __ldg(z4 + k);
                const uint32_t w4[4] = {t4.x, t4.y, t4.z, t4.w};
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                  zv[8 * k + 2 * m] = __uint_as_float(w4[m] << 16);
                  zv[8 * k + 2 * m + 1] = __uint_as_float(w4[m] & 0xffff0000u);
                }
              }
            }
#pragma unroll
            for (int e = 0; e < 32; ++e) acc[e] = fmaf(zv[e], __uint_as_float(o[e]) * inv_o, acc[e]);
            if (SAVE) {
              float* us = a.osave + (bi * p.H + h) * (size_t)(p.Dv + 3 * p.Q + RCz) + p.Dv + 3 * p.Q + rr * Cz + c0;
#pragma unroll
              for (int e = 0; e < 32; ++e) us[e] = __uint_as_float(o[e]) * inv_o;
            }
          }
        }
        if (in_range && !empty) put_run32(frow, p.Wh8, p.f32, pcol + c0, acc);
      }
    }
  }
  ttr.ev(47);
  // ---------------------------------------------------------------- teardown
  ttr.ev(43);
  tc_fence_before();
  __syncthreads();
  ttr.ev(44);
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

cudaError_t launch_core(const Plan& p, const Inputs& in, const Work& w, const Outputs& out,
                        const CUtensorMap& tmQ, const CUtensorMap& tmKH, const CUtensorMap& tmVH,
                        const CUtensorMap& tmZ, const DeviceCtl& ctl, cudaStream_t s, float* osave) {
  CoreArgs a;
  a.p = p;
  a.kvec = w.kvec; a.qvec = w.qvec; a.QP = w.QP; a.KP = w.KP; a.orig = w.orig; a.flag = w.flag;
  a.mask = in.mask; a.pair_mask = in.pair_mask; a.raw = in.raw;
  a.rot = in.rot; a.trans = in.trans; a.z1 = in.z1; a.feat = w.feat; a.rowflag = w.rowflag;
  a.local_points = out.local_points; a.eps = in.eps;
  a.stats = w.stats; a.lse = out.lse;
  a.status = ctl.status; a.timeout_ns = ctl.timeout_ns;
  a.trace = ctl.trace; a.trace_cta = ctl.trace_cta;
  a.osave = osave;
  dim3 grid(cdiv(p.row1, kTile) - p.row0 / kTile, p.H, p.B);   // the query tiles of the row range
  auto kfn = p.f32 ? (osave ? fipa_core_kernel<true, false, true> : fipa_core_kernel<true, false, false>)
                   : (p.vbuf ? (osave ? fipa_core_kernel<false, true, true> : fipa_core_kernel<false, true, false>)
                             : (osave ? fipa_core_kernel<false, false, true> : fipa_core_kernel<false, false, false>));
  cudaError_t e = allow_max_smem(reinterpret_cast<const void*>(kfn));
  if (e != cudaSuccess) return e;
  kfn<<<grid, 256, p.core_smem, s>>>(tmQ, tmKH, tmVH, tmZ, a);
  return cudaGetLastError();
}

}  // namespace fipa
