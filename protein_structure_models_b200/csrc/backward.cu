// backward.cu -- backward pass of the fused IPA core on tcgen05 (training).
//
// Gradients of <d_update, update> + <d_local, local_points> with respect to
// every floating input of the forward defined on the BioTorch page "Invariant
// point attention (IPA)", section "Required behavior" (whose test suite grades
// gradients, section "Starter code").  The forward has been recomputed by the
// lift and the fused core (which also saved the normalised aggregates
// O = [o_scalar | G | U] of every row); its lifted rows, row statistics (M, l),
// per-key / per-row fp32 terms and group origins are in the workspace.
//
// With the true (origin-free) global points a_i (query), b_j (key), g_j (value):
//   dO_i  = [d o_scalar | dG | dU],  dU[r,c] = z1[i,r,c] d o_pair[c]
//   D_i   = dO_i . O_i,   dP_ij = dO_i . [v_j | g_j | z2_j],   dS_ij = P_ij (dP_ij - D_i)
//   dq_i  = sum_j dS_ij k_j / sqrt(3D),      dk_j = sum_i dS_ij q_i / sqrt(3D)
//   da_i  = 2 g sum_j dS_ij (b_j - a_i),     db_j = 2 g sum_i dS_ij (a_i - b_j)
//   du_i  = sum_j dS_ij z2_j  (u = z1 Wb / sqrt(3)),   dz2_j += sum_i dS_ij u_i + P_ij dU_i
//   dv_j  = sum_i P_ij d o_scalar_i,         dg_j = sum_i P_ij dG_i
//   dg_h  = -sum_ij dS_ij |a_i - b_j|^2      (g = 1/2 softplus(raw) sqrt(2/(27P)))
// The coordinate sums run on relative coordinates a' = a - o, b' = b - o (o
// the 32-residue group origins of plan.h) with the origin differences taken
// in fp32, exactly as the forward does.
#include "bwd_plan.h"
#include "kernels.h"
#include "sm100.cuh"

namespace fipa {
namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kInvSqrt3 = 0.57735026918962576f;

struct BwdArgs {
  Plan p;
  BwdPlan bp;
  const void *q_pts, *k_pts, *v_pts, *rot, *trans, *z1, *Wb, *raw, *w_out;
  const uint8_t* mask;
  const uint8_t* pair_mask;
  float eps;
  const float* d_update;
  const float* d_local;             // may be null (zero cotangent)
  const float4 *kvec, *qvec, *orig;
  const int* flag;
  const float2* stats;
  const uint8_t* rowflag;
  float* osave;
  float* dfeat;
  __nv_bfloat16* fhi;               // feature rows [F | 1 | 0..] as bfloat16 hi / lo (the dw_out operand)
  __nv_bfloat16* flo;
  __half* dO;
  float4* dvec;
  float* rloc;
  float* dz1u;
  float* qres;
  float* du;
  float* kres;
  float* dz2h;
  float* dwpart;
  float* wbpart;
  float* gpart;
  BwdGrads g;
  int* status;
  unsigned long long timeout_ns;
};

// An input value as float: float32 or bfloat16 inputs (Plan::in_f32).
__device__ __forceinline__ float ldi(const void* p, size_t i, int f32) {
  return f32 ? static_cast<const float*>(p)[i] : __bfloat162float(static_cast<const __nv_bfloat16*>(p)[i]);
}

// ------------------------------------------------------------------ dw_out reduce
// The dense products dfeat = d_update w_out^T and features^T d_update run on
// the tensor cores (bgemm.cu); the latter's row splits are added here in order.
// dw_out[f, c] = sum_z part[z, f, c] (f < F), db_out[c] = sum_z part[z, F, c].
__global__ void bwd_dw_reduce_kernel(const float* __restrict__ part, float* __restrict__ dw, float* __restrict__ db,
                                     int F, int Fp, int Cout, int ks) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= (F + 1) * Cout) return;
  const int f = e / Cout, c = e - f * Cout;
  float s = 0.f;
  for (int z = 0; z < ks; ++z) s += part[((size_t)z * Fp + f) * Cout + c];
  if (f < F) dw[(size_t)f * Cout + c] = s;
  else db[c] = s;
}

// ------------------------------------------------------------------ prep
// One CTA per residue (b, i): the cotangent of the value aggregates,
//   d local = (dx, dy, dz) + d len * local / len + d_local,  dG = R_i d local,
//   dU[r,c] = z1[i,r,c] d o_pair[c],
// written as the fp16 dO row of every head [d o_s | dG | dG | 0 | dU | 0]
// (the value operand's layout [v | g' hi | g' lo | 0 | z2 | 0]), with
// D = fp16(dO) . O and sG = sum_q fp16(dG_q); the parts of the chain rule that
// stay on this residue (local = R^T (G - t): dR += (G - t) (x) d local,
// dt -= dG; dz1 += U d o_pair), and the fp32 feature row for dw_out.
// Feature value v at flat index idx of the bfloat16 hi / lo feature rows.
__device__ __forceinline__ void put_feat(const BwdArgs& a, size_t idx, float v) {
  const __nv_bfloat16 hv = __float2bfloat16_rn(v);
  a.fhi[idx] = hv;
  a.flo[idx] = __float2bfloat16_rn(v - __bfloat162float(hv));
}

// WPR warps per residue (b, i): 1 (a CTA holds `wpc` residues; many
// residues) or 8 (one residue per CTA; few residues, more threads each).  The
// group's shared memory holds dG [H][3Q]; sums over a residue's items (the
// frame terms, D) are per-thread partial sums added in a fixed order (warp
// shuffle tree, then the warps in order).
template <int WPR>
__global__ void __launch_bounds__(256) bwd_prep_kernel(const BwdArgs a, int wpc) {
  const Plan& p = a.p;
  const BwdPlan& bp = a.bp;
  extern __shared__ float psm[];
  constexpr int T = 32 * WPR;                                 // threads per residue
  const int H = p.H, Dv = p.Dv, Q = p.Q, Cz = p.Cz, RCz = bp.RCz, F = p.F;
  const int HDv = H * Dv, HQ = H * Q, pairblk = HDv + 4 * HQ;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int grp = WPR == 1 ? warp : 0;                        // residue slot in the CTA
  const int gw = WPR == 1 ? 0 : warp;                         // warp within the residue
  const int gt = gw * 32 + lane;                              // thread within the residue
  const size_t bi = (size_t)blockIdx.x * wpc + grp;
  if (bi >= (size_t)p.B * p.N) return;                       // whole groups only
  const int b = (int)(bi / p.N), i = (int)(bi - (size_t)b * p.N);
  float* sdG = psm + (size_t)grp * rup(H * 3 * Q, 4);        // [H][3Q]
  float* red = psm + (size_t)(WPR == 1 ? wpc : 1) * rup(H * 3 * Q, 4);   // [WPR][12] (WPR > 1)
  auto group_sync = [&]() {
    if (WPR == 1) __syncwarp();
    else __syncthreads();
  };
  const float* df = a.dfeat + bi * F;
  const size_t fr = bi * bp.Fp;
  if (a.rowflag[bi] == 0) {                                   // uniform over the group
    for (int h = gw; h < H; h += WPR) {
      uint4* drow = reinterpret_cast<uint4*>(a.dO + ((size_t)(b * H + h) * p.N + i) * bp.Vw);
      for (int c = lane; c < bp.Vw / 8; c += 32) drow[c] = make_uint4(0u, 0u, 0u, 0u);
      if (lane == 0) a.dvec[(size_t)(b * H + h) * p.N + i] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    if (gt < 12) a.rloc[bi * 12 + gt] = 0.f;
    for (int e = gt; e < RCz; e += T) a.dz1u[bi * RCz + e] = 0.f;
    for (int e = gt; e < bp.Fp; e += T) put_feat(a, fr + e, 0.f);
    return;
  }
  float R[9], t[3];
#pragma unroll
  for (int e = 0; e < 9; ++e) R[e] = ldi(a.rot, bi * 9 + e, a.p.in_f32);
#pragma unroll
  for (int e = 0; e < 3; ++e) t[e] = ldi(a.trans, bi * 3 + e, a.p.in_f32);
  // points: (h, q) items over the lanes
  float acc[12];
#pragma unroll
  for (int k = 0; k < 12; ++k) acc[k] = 0.f;
  for (int it = gt; it < HQ; it += T) {
    const int h = it / Q, q = it - h * Q;
    const float* G = a.osave + (bi * H + h) * (size_t)bp.Osw + Dv + 3 * q;
    const float gt[3] = {G[0] - t[0], G[1] - t[1], G[2] - t[2]};
    float loc[3];
#pragma unroll
    for (int x = 0; x < 3; ++x) loc[x] = R[x] * gt[0] + R[3 + x] * gt[1] + R[6 + x] * gt[2];
    const float len = sqrtf(loc[0] * loc[0] + loc[1] * loc[1] + loc[2] * loc[2] + a.eps);
    const float dlen = __ldg(df + HDv + 3 * HQ + h * Q + q);
    float dl[3];
#pragma unroll
    for (int x = 0; x < 3; ++x) {
      dl[x] = __ldg(df + HDv + x * HQ + h * Q + q) + dlen * loc[x] / len;
      if (a.d_local != nullptr) dl[x] += a.d_local[((bi * H + h) * Q + q) * 3 + x];
    }
#pragma unroll
    for (int y = 0; y < 3; ++y) {
      const float dG = R[3 * y] * dl[0] + R[3 * y + 1] * dl[1] + R[3 * y + 2] * dl[2];
      sdG[h * 3 * Q + 3 * q + y] = dG;
      acc[9 + y] -= dG;
#pragma unroll
      for (int x = 0; x < 3; ++x) acc[3 * y + x] += gt[y] * dl[x];
    }
    put_feat(a, fr + HDv + h * Q + q, loc[0]);
    put_feat(a, fr + HDv + HQ + h * Q + q, loc[1]);
    put_feat(a, fr + HDv + 2 * HQ + h * Q + q, loc[2]);
    put_feat(a, fr + HDv + 3 * HQ + h * Q + q, len);
  }
  float mine = 0.f;
#pragma unroll
  for (int k = 0; k < 12; ++k) {
    float v = acc[k];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == k) mine = v;
  }
  if (WPR == 1) {
    if (lane < 12) a.rloc[bi * 12 + lane] = mine;
  } else {
    if (lane < 12) red[gw * 12 + lane] = mine;
  }
  group_sync();                                               // dG rows and warp sums visible
  if (WPR > 1 && gt < 12) {
    float v = 0.f;
    for (int w = 0; w < WPR; ++w) v += red[w * 12 + gt];
    a.rloc[bi * 12 + gt] = v;
  }
  // dO rows, D and sG: heads over the group's warps
  for (int h = gw; h < H; h += WPR) {
    const float* Oh = a.osave + (bi * H + h) * (size_t)bp.Osw;
    uint4* drow = reinterpret_cast<uint4*>(a.dO + ((size_t)(b * H + h) * p.N + i) * bp.Vw);
    float Dp = 0.f;
    for (int c8 = lane; c8 < bp.Vw / 8; c8 += 32) {
      uint32_t w[4];
#pragma unroll
      for (int e2 = 0; e2 < 4; ++e2) {
        float xv[2], ov[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int c = c8 * 8 + e2 * 2 + u;
          float x = 0.f, o = 0.f;
          if (c < Dv) {
            x = __ldg(df + h * Dv + c);
            o = Oh[c];
          } else if (c >= p.Dv8 && c < p.Dv8 + 3 * Q) {
            x = sdG[h * 3 * Q + c - p.Dv8];
            o = Oh[Dv + c - p.Dv8];
          } else if (c >= p.Dv8 + p.Q38 && c < p.Dv8 + p.Q38 + 3 * Q) {
            x = sdG[h * 3 * Q + c - p.Dv8 - p.Q38];       // second copy: meets g' lo, not part of D
          } else if (c >= p.VHp && c < p.VHp + RCz) {
            const int rc = c - p.VHp, cc = rc % Cz;
            x = ldi(a.z1, bi * RCz + rc, a.p.in_f32) * __ldg(df + pairblk + h * Cz + cc);
            o = Oh[Dv + 3 * Q + rc];
          }
          xv[u] = x;
          ov[u] = o;
        }
        const __half2 hv = __floats2half2_rn(xv[0], xv[1]);
        const float2 fv = __half22float2(hv);
        Dp = fmaf(fv.x, ov[0], Dp);
        Dp = fmaf(fv.y, ov[1], Dp);
        w[e2] = *reinterpret_cast<const uint32_t*>(&hv);
      }
      drow[c8] = make_uint4(w[0], w[1], w[2], w[3]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) Dp += __shfl_xor_sync(0xffffffffu, Dp, o);
    float sg = 0.f;
    if (lane < 3)
      for (int q = 0; q < Q; ++q) sg += __half2float(__float2half_rn(sdG[h * 3 * Q + 3 * q + lane]));
    const float sx = __shfl_sync(0xffffffffu, sg, 0), sy = __shfl_sync(0xffffffffu, sg, 1),
                sz = __shfl_sync(0xffffffffu, sg, 2);
    if (lane == 0) a.dvec[(size_t)(b * H + h) * p.N + i] = make_float4(Dp, sx, sy, sz);
  }
  // dz1 from the pair aggregate, and the scalar / pair feature blocks
  for (int rc = gt; rc < RCz; rc += T) {
    const int cc = rc % Cz;
    float s = 0.f;
    for (int h = 0; h < H; ++h)
      s = fmaf(a.osave[(bi * H + h) * (size_t)bp.Osw + Dv + 3 * Q + rc], __ldg(df + pairblk + h * Cz + cc), s);
    a.dz1u[bi * RCz + rc] = s;
  }
  for (int e = gt; e < HDv; e += T) {
    const int h = e / Dv, d = e - h * Dv;
    put_feat(a, fr + e, a.osave[(bi * H + h) * (size_t)bp.Osw + d]);
  }
  for (int e = gt; e < H * Cz; e += T) {
    const int h = e / Cz, c = e - h * Cz;
    const float* U = a.osave + (bi * H + h) * (size_t)bp.Osw + Dv + 3 * Q;
    float s = 0.f;
    for (int r = 0; r < p.R; ++r) s = fmaf(ldi(a.z1, bi * RCz + r * Cz + c, a.p.in_f32), U[r * Cz + c], s);
    put_feat(a, fr + pairblk + e, s);
  }
  for (int e = F + gt; e < bp.Fp; e += T) put_feat(a, fr + e, e == F ? 1.f : 0.f);
}

// ------------------------------------------------------------------ shared pieces
// Bounded wait that ignores the abort flag (used only to drain in-flight work).
__device__ __forceinline__ void bwd_drain_wait(uint64_t* bar, uint32_t parity, uint64_t timeout_ns) {
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > timeout_ns) break;
  }
}

__device__ __forceinline__ float bwd_raw(const BwdArgs& a, int h) { return ldi(a.raw, h, a.p.in_f32); }

// The TMA ring shared by the producer and the MMA thread of both kernels.
struct Ring {
  uint64_t* full;
  uint64_t* empty;
  uint8_t* base;
  int nst;
  int st = 0;
  uint32_t ph = 0;
  __device__ __forceinline__ uint8_t* slot() const { return base + st * kChunkBytes; }
  __device__ __forceinline__ void next() {
    if (++st == nst) { st = 0; ph ^= 1u; }
  }
};

// Bit e: pair-mask entry first + e (stride `stride` bytes apart) allowed; 0 past
// N.  Every load is issued unconditionally (an index past N reads entry 0) and
// the results combine afterwards, so the 32 loads are in flight together.
__device__ __forceinline__ uint32_t pair_bits32(const uint8_t* base, size_t stride, int first, int N) {
  uint32_t v[32];
#pragma unroll
  for (int e = 0; e < 32; ++e) {
    const int x = first + e;
    v[e] = __ldg(base + (size_t)(x < N ? x : 0) * stride);
  }
  uint32_t bits = 0;
#pragma unroll
  for (int e = 0; e < 32; ++e) bits |= (first + e < N && v[e] != 0u) ? (1u << e) : 0u;
  return bits;
}
// The 128 bits of a tile, out of line: the loads' registers stay out of the
// kernels' main loops (the pair mask is the uncommon case).
__device__ __noinline__ uint4 pair_bits128(const uint8_t* base, size_t stride, int first, int N) {
  return make_uint4(pair_bits32(base, stride, first, N), pair_bits32(base, stride, first + 32, N),
                    pair_bits32(base, stride, first + 64, N), pair_bits32(base, stride, first + 96, N));
}

// ------------------------------------------------------------------ q side
// One CTA per (query tile, head, sample), as the forward core.  Per key tile s:
//   QK(s): S = Qhat Khat^T (u hi resident, u lo streamed with the z2 chunks)
//   DP(s): dP = dO Vhat^T into the same TMEM columns once S has been read
//   DQ(s): dQhat += dS [KH | Z] with dS (fp16) in TMEM as the A operand
// issued as QK(0) DP(0) [QK(s+1) DQ(s) DP(s+1)]..., so the next logits are
// computed while the softmax warps form dS.
constexpr int kQBarFull = 0, kQBarEmpty = 64, kQBarRes = 128, kQBarSFull = 136, kQBarSRead = 144,
              kQBarDPFull = 152, kQBarDPRead = 160, kQBarDSFull = 168, kQBarDQDone = 176, kQBarKtFull = 184,
              kQBarKtEmpty = 200, kQBarDrain = 216;
constexpr int kQOk = 256, kQMisc = 384, kQKt = 1024, kQTiles = 5120;

__global__ void __launch_bounds__(256, 1)
bwd_q_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmKH,
             const __grid_constant__ CUtensorMap tmVH, const __grid_constant__ CUtensorMap tmZ,
             const __grid_constant__ CUtensorMap tmdO, const BwdArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const Plan& p = a.p;
  const BwdPlan& bp = a.bp;
  uint8_t* sQ = smem;                                  // QH + u hi chunks of the query tile
  uint8_t* sO = sQ + bp.nQr * kChunkBytes;             // dO chunks of the query tile
  uint8_t* sRing = sO + bp.nOc * kChunkBytes;
  uint8_t* tail = sRing + bp.q_nst * kChunkBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(tail + kQBarFull);
  uint64_t* empty = reinterpret_cast<uint64_t*>(tail + kQBarEmpty);
  uint64_t* res_full = reinterpret_cast<uint64_t*>(tail + kQBarRes);
  uint64_t* s_full = reinterpret_cast<uint64_t*>(tail + kQBarSFull);
  uint64_t* s_read = reinterpret_cast<uint64_t*>(tail + kQBarSRead);
  uint64_t* dp_full = reinterpret_cast<uint64_t*>(tail + kQBarDPFull);
  uint64_t* dp_read = reinterpret_cast<uint64_t*>(tail + kQBarDPRead);
  uint64_t* ds_full = reinterpret_cast<uint64_t*>(tail + kQBarDSFull);
  uint64_t* dq_done = reinterpret_cast<uint64_t*>(tail + kQBarDQDone);
  uint64_t* kt_full = reinterpret_cast<uint64_t*>(tail + kQBarKtFull);
  uint64_t* kt_empty = reinterpret_cast<uint64_t*>(tail + kQBarKtEmpty);
  uint64_t* drain = reinterpret_cast<uint64_t*>(tail + kQBarDrain);
  float4* okbuf = reinterpret_cast<float4*>(tail + kQOk);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tail + kQMisc);
  int* abort_flag = reinterpret_cast<int*>(tail + kQMisc + 4);
  int* ntiles = reinterpret_cast<int*>(tail + kQMisc + 8);
  float* ktbuf = reinterpret_cast<float*>(tail + kQKt);
  uint16_t* tiles = reinterpret_cast<uint16_t*>(tail + kQTiles);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int bh = b * p.H + h;
  const int N = p.N, nT = p.nT;

  if (threadIdx.x == 0) {
    for (int s = 0; s < bp.q_nst; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    mbar_init(res_full, 1);
    mbar_init(s_full, 1);
    mbar_init(s_read, 128);
    mbar_init(dp_full, 1);
    mbar_init(dp_read, 128);
    mbar_init(ds_full, 128);
    mbar_init(dq_done, 1);
    mbar_init(&kt_full[0], 64);
    mbar_init(&kt_full[1], 64);
    mbar_init(&kt_empty[0], 128);
    mbar_init(&kt_empty[1], 128);
    mbar_init(drain, 1);
    fence_mbar_init();
    *abort_flag = 0;
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
  const int nKH = p.nKH, nZ = p.nZ, nVH = p.nVH, nqz = p.nqz;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && nkt > 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmKH);
      tma_prefetch_desc(&tmVH);
      tma_prefetch_desc(&tmZ);
      tma_prefetch_desc(&tmdO);
      mbar_arrive_expect_tx(res_full, (uint32_t)((bp.nQr + bp.nOc) * kChunkBytes));
      for (int c = 0; c < bp.nQr; ++c) tma_load_3d(sQ + c * kChunkBytes, &tmQ, res_full, c * kChunk, qt * kTile, bh);
      for (int c = 0; c < bp.nOc; ++c) tma_load_3d(sO + c * kChunkBytes, &tmdO, res_full, c * kChunk, qt * kTile, bh);
      Ring rg{full, empty, sRing, bp.q_nst};
      bool ok = true;
      uint32_t issued = 0;
      auto push = [&](const CUtensorMap* tm, int c0, int c1, int c2) {
        if (!ok) return;
        if (!mbar_wait(&empty[rg.st], rg.ph ^ 1u, wc, 21)) { ok = false; return; }
        mbar_arrive_expect_tx(&full[rg.st], kChunkBytes);
        tma_load_3d(rg.slot(), tm, &full[rg.st], c0, c1, c2);
        ++issued;
        rg.next();
      };
      auto push_qk = [&](int kt) {
        for (int c = 0; c < nZ; ++c) {
          push(&tmZ, c * kChunk, kt * kTile, b);
          for (int qz = 1; qz < nqz; ++qz) push(&tmQ, (nKH + qz * nZ + c) * kChunk, qt * kTile, bh);
        }
        for (int c = 0; c < nKH; ++c) push(&tmKH, c * kChunk, kt * kTile, bh);
      };
      auto push_dp = [&](int kt) {
        for (int c = 0; c < nVH; ++c) push(&tmVH, c * kChunk, kt * kTile, bh);
        for (int c = 0; c < nZ; ++c) push(&tmZ, c * kChunk, kt * kTile, b);
      };
      auto push_dq = [&](int kt) {
        for (int c = 0; c < nKH; ++c) push(&tmKH, c * kChunk, kt * kTile, bh);
        for (int c = 0; c < nZ; ++c) push(&tmZ, c * kChunk, kt * kTile, b);
      };
      push_qk(tiles[0]);
      push_dp(tiles[0]);
      for (int s = 0; s < nkt && ok; ++s) {
        if (s + 1 < nkt) push_qk(tiles[s + 1]);
        push_dq(tiles[s]);
        if (s + 1 < nkt) push_dp(tiles[s + 1]);
      }
      if (*abort_flag) {
        bwd_drain_wait(res_full, 0, a.timeout_ns);
        const uint32_t last = issued < (uint32_t)bp.q_nst ? issued : (uint32_t)bp.q_nst;
        for (uint32_t k = 0; k < last; ++k) {
          const uint32_t n = issued - 1 - k;
          bwd_drain_wait(&full[n % bp.q_nst], (n / bp.q_nst) & 1u, a.timeout_ns);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && nkt > 0) {
      bool ok = mbar_wait(res_full, 0, wc, 22);
      tc_fence_after();
      Ring rg{full, empty, sRing, bp.q_nst};
      const uint32_t idS = idesc_f16(128, 128, 0, 0);
      const uint32_t sQa = smem_u32(sQ), sOa = smem_u32(sO);
      auto take = [&](int site) -> int {
        if (!mbar_wait(&full[rg.st], rg.ph, wc, site)) return -1;
        tc_fence_after();
        const int st = rg.st;
        rg.next();
        return st;
      };
      const uint32_t ringa = smem_u32(sRing);
      auto mma_qk = [&]() -> bool {
        for (int c = 0; c < nZ; ++c) {
          const int sz = take(23);
          if (sz < 0) return false;
          const uint32_t bz = ringa + sz * kChunkBytes;
          const uint32_t ah = sQa + (nKH + c) * kChunkBytes;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ss(tmem, desc_kmajor_sw128(ah + kk * 32), desc_kmajor_sw128(bz + kk * 32), idS, (c | kk) != 0);
          for (int qz = 1; qz < nqz; ++qz) {
            const int sl = take(23);
            if (sl < 0) return false;
            const uint32_t al = ringa + sl * kChunkBytes;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_ss(tmem, desc_kmajor_sw128(al + kk * 32), desc_kmajor_sw128(bz + kk * 32), idS, 1u);
            tc_commit(&empty[sl]);
          }
          tc_commit(&empty[sz]);
        }
        for (int c = 0; c < nKH; ++c) {
          const int sk = take(23);
          if (sk < 0) return false;
          const uint32_t bk = ringa + sk * kChunkBytes, ak = sQa + c * kChunkBytes;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ss(tmem, desc_kmajor_sw128(ak + kk * 32), desc_kmajor_sw128(bk + kk * 32), idS, 1u);
          tc_commit(&empty[sk]);
        }
        tc_commit(s_full);
        return true;
      };
      auto mma_dp = [&]() -> bool {
        for (int c = 0; c < bp.nOc; ++c) {
          const int sv = take(24);
          if (sv < 0) return false;
          const uint32_t bv = ringa + sv * kChunkBytes, ao = sOa + c * kChunkBytes;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ss(tmem, desc_kmajor_sw128(ao + kk * 32), desc_kmajor_sw128(bv + kk * 32), idS, (c | kk) != 0);
          tc_commit(&empty[sv]);
        }
        tc_commit(dp_full);
        return true;
      };
      // dQhat += dS [KH | Z]: chunks in consecutive ring slots form one MMA of
      // N = 64 x run (up to 4), into consecutive 64-column blocks of dQhat
      auto mma_dq = [&](int s) -> bool {
        const int nch = nKH + nZ;
        for (int c = 0; c < nch;) {
          int run = nch - c;
          if (run > 4) run = 4;
          if (run > rg.nst - rg.st) run = rg.nst - rg.st;
          for (int u = 0; u < run; ++u)
            if (!mbar_wait(&full[rg.st + u], rg.ph, wc, 25)) return false;
          tc_fence_after();
          const uint32_t bk = ringa + rg.st * kChunkBytes;
          const uint32_t dcol = tmem + (uint32_t)(bp.tmDQ + c * kChunk);
          const uint32_t idR = idesc_f16(128, 64 * run, 0, 1);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ts(dcol, tmem + (uint32_t)bp.tmDS + kk * 8, desc_mnmajor_sw128(bk + kk * 2048, kChunkBytes), idR,
                   (s > 0 || kk > 0) ? 1u : 0u);
          for (int u = 0; u < run; ++u) tc_commit(&empty[rg.st + u]);
          rg.st += run;
          if (rg.st == rg.nst) { rg.st = 0; rg.ph ^= 1u; }
          c += run;
        }
        tc_commit(dq_done);
        return true;
      };
      if (ok) ok = mma_qk();
      if (ok) ok = mbar_wait(s_read, 0, wc, 26);
      if (ok) { tc_fence_after(); ok = mma_dp(); }
      for (int s = 0; ok && s < nkt; ++s) {
        if (s + 1 < nkt) {
          if (!mbar_wait(dp_read, s & 1, wc, 27)) break;
          tc_fence_after();
          if (!mma_qk()) break;
        }
        if (!mbar_wait(ds_full, s & 1, wc, 28)) break;
        tc_fence_after();
        if (!mma_dq(s)) break;
        if (s + 1 < nkt) {
          if (!mbar_wait(s_read, (s + 1) & 1, wc, 29)) break;
          tc_fence_after();
          if (!mma_dp()) break;
        }
      }
      tc_commit(drain);
      bwd_drain_wait(drain, 0, a.timeout_ns);
    }
  } else if (warp == 2 || warp == 3) {
    // ------------------------------------------------------------ per-key terms
    // kterm[s][j] = -g sum_p |b'_p|^2 + 2g D_sj . sum_p b'_p (-inf for a masked or
    // absent key), D_sj = origin of query group s - origin of key j's group
    const int tt = threadIdx.x - 64;
    const float g = point_weight(bwd_raw(a, h), p.P);
    float4 oq[4];
#pragma unroll
    for (int sq = 0; sq < 4; ++sq) oq[sq] = a.orig[(size_t)b * p.nG + qt * 4 + sq];
    for (int s = 0; s < nkt; ++s) {
      const int kb = s & 1;
      const bool okw = mbar_wait(&kt_empty[kb], ((s >> 1) & 1) ^ 1, wc, 30);
      if (!__all_sync(0xffffffffu, okw)) break;
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
          ktbuf[(kb * 4 + sq) * kTile + e] = kv.x + 2.f * g * (dx * kv.y + dy * kv.z + dz * kv.w);
        }
      }
      mbar_arrive(&kt_full[kb]);
    }
  } else {
    // ------------------------------------------------------------ softmax warps
    // thread = query row = TMEM lane.  P = 2^((S + kterm + rc) log2e - M) / l from
    // the forward's row statistics; dS = P (dP + sG . o_t - D) rounded to fp16
    // (the value the dQhat product uses; every sum below adds the rounded values).
    const int wq = warp - 4;
    const int r = wq * 32 + lane;
    const int i = qt * kTile + r;
    const bool in_range = i < N;
    const bool row_valid = in_range && a.mask[(size_t)b * N + i] != 0;
    const float2 st = in_range ? a.stats[(size_t)bh * N + i] : make_float2(0.f, 0.f);
    const float invl = (row_valid && st.y > 0.f) ? 1.f / st.y : 0.f;
    const float4 qv = in_range ? a.qvec[(size_t)bh * N + i] : make_float4(0.f, 0.f, 0.f, 0.f);
    const float4 dvv = in_range ? a.dvec[(size_t)bh * N + i] : make_float4(0.f, 0.f, 0.f, 0.f);
    const float4 oqs = a.orig[(size_t)b * p.nG + qt * 4 + wq];
    const float g = point_weight(bwd_raw(a, h), p.P);
    const uint32_t trow = tmem + ((uint32_t)(wq * 32) << 16);
    const uint8_t* pmrow = (a.pair_mask != nullptr && in_range) ? a.pair_mask + ((size_t)b * N + i) * N : nullptr;
    float rs = 0.f, Wx = 0.f, Wy = 0.f, Wz = 0.f, E = 0.f;
    bool ok = true;
    for (int s = 0; s < nkt; ++s) {
      const int kt = tiles[s];
      const int kb = s & 1;
      ok = mbar_wait(s_full, s & 1, wc, 31);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      tc_fence_after();
      uint32_t sv[4][32];
      tmem_ld32(trow + 0, sv[0]);
      tmem_ld32(trow + 32, sv[1]);
      tmem_ld32(trow + 64, sv[2]);
      tmem_ld32(trow + 96, sv[3]);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(s_read);
      ok = mbar_wait(&kt_full[kb], (s >> 1) & 1, wc, 32);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      float4 okg[4];
      float rc[4];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        okg[t] = okbuf[kb * 4 + t];
        const float dx = oqs.x - okg[t].x, dy = oqs.y - okg[t].y, dz = oqs.z - okg[t].z;
        rc[t] = -g * ((float)p.P * (dx * dx + dy * dy + dz * dz) + 2.f * (dx * qv.x + dy * qv.y + dz * qv.z));
      }
      const float* ktw = ktbuf + (kb * 4 + wq) * kTile;
      // a forbidden pair gets the logit -inf in a pass of its own, so that the
      // loop below has no branch (absent or masked keys have kterm -inf already)
      if (pmrow != nullptr) {
        const uint4 b4 = pair_bits128(pmrow, 1, kt * kTile, N);
        const uint32_t bw[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
        for (int t = 0; t < 4; ++t)
#pragma unroll
          for (int e = 0; e < 32; ++e)
            sv[t][e] = ((bw[t] >> e) & 1u) ? sv[t][e] : __float_as_uint(-INFINITY);
      }
      const bool allow = invl > 0.f;
      uint32_t pk[2][32];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const float mb = allow ? st.x - rc[t] * kLog2e : 0.f;
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          float pv[2];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int jl = t * 32 + e + u;
            const float x = __uint_as_float(sv[t][e + u]) + ktw[jl];
            pv[u] = allow ? ex2_approx(fmaf(x, kLog2e, -mb)) * invl : 0.f;
          }
          pk[t >> 1][(t & 1) * 16 + e / 2] = pack_half2(pv[0], pv[1]);
        }
      }
      ok = mbar_wait(dp_full, s & 1, wc, 33);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      tc_fence_after();
      tmem_ld32(trow + 0, sv[0]);
      tmem_ld32(trow + 32, sv[1]);
      tmem_ld32(trow + 64, sv[2]);
      tmem_ld32(trow + 96, sv[3]);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(dp_read);
      uint32_t dk[2][32];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        // dP against the true value points: + sG . o_t (the MMA used g' = g - o_t)
        const float sgo = dvv.y * okg[t].x + dvv.z * okg[t].y + dvv.w * okg[t].z - dvv.x;
        float rst = 0.f, Ek = 0.f;
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const float2 pp = __half22float2(*reinterpret_cast<const __half2*>(&pk[t >> 1][(t & 1) * 16 + e / 2]));
          const float d0 = pp.x * (__uint_as_float(sv[t][e]) + sgo);
          const float d1 = pp.y * (__uint_as_float(sv[t][e + 1]) + sgo);
          const __half2 hd = __floats2half2_rn(d0, d1);
          const float2 fd = __half22float2(hd);
          rst += fd.x + fd.y;
          if (pp.x != 0.f) Ek = fmaf(fd.x, ktw[t * 32 + e], Ek);
          if (pp.y != 0.f) Ek = fmaf(fd.y, ktw[t * 32 + e + 1], Ek);
          dk[t >> 1][(t & 1) * 16 + e / 2] = *reinterpret_cast<const uint32_t*>(&hd);
        }
        E += Ek + rc[t] * rst;
        rs += rst;
        Wx = fmaf(rst, okg[t].x, Wx);
        Wy = fmaf(rst, okg[t].y, Wy);
        Wz = fmaf(rst, okg[t].z, Wz);
      }
      mbar_arrive(&kt_empty[kb]);
      if (s > 0) {
        ok = mbar_wait(dq_done, (s - 1) & 1, wc, 34);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        tc_fence_after();
      }
      tmem_st32(trow + (uint32_t)bp.tmDS, dk[0]);
      tmem_st32(trow + (uint32_t)bp.tmDS + 32, dk[1]);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(ds_full);
    }
    if (ok && nkt > 0) {
      ok = mbar_wait(dq_done, (nkt - 1) & 1, wc, 35);
      ok = __all_sync(0xffffffffu, ok);
      tc_fence_after();
    }
    // results of this row: [sum dS k | X | rs | W | E] and du = sum_j dS_ij z2_j.
    // tcgen05.ld is warp-collective: every lane loads, only rows in range store.
    const bool aborted = __any_sync(0xffffffffu, *abort_flag != 0);
    const bool wr = in_range && !aborted;
    const bool have = nkt > 0 && !aborted;
    float* qr = a.qres + ((size_t)bh * N + (in_range ? i : 0)) * bp.Kr;
    float* dur = a.du + ((size_t)bh * N + (in_range ? i : 0)) * bp.RCz;
    float xlo[3 * kMaxPts];
#pragma unroll 1
    for (int x = 0; x < 3 * p.P; ++x) xlo[x] = 0.f;
    for (int c0 = 0; c0 < 64 * (nKH + nZ); c0 += 32) {
      uint32_t o[32];
      if (have) {
        tmem_ld32(trow + (uint32_t)(bp.tmDQ + c0), o);
        tmem_ld_wait();
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) o[e] = 0u;
      }
      if (wr) {
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int c = c0 + e;
          const float v = __uint_as_float(o[e]);
          if (c < p.D) {
            qr[c] = v;
          } else if (c >= p.D8 && c < p.D8 + 3 * p.P) {
            qr[p.D + c - p.D8] = v;                                     // b' hi part of X
          } else if (c >= p.D8 + p.P38 && c < p.D8 + p.P38 + 3 * p.P) {
            xlo[c - p.D8 - p.P38] = v;                                  // b' lo part of X
          } else if (c >= p.KHp && c < p.KHp + bp.RCz) {
            dur[c - p.KHp] = v;
          }
        }
      }
    }
    if (wr) {
      for (int x = 0; x < 3 * p.P; ++x) qr[p.D + x] += xlo[x];
      qr[p.D + 3 * p.P] = rs;
      qr[p.D + 3 * p.P + 1] = Wx;
      qr[p.D + 3 * p.P + 2] = Wy;
      qr[p.D + 3 * p.P + 3] = Wz;
      qr[p.D + 3 * p.P + 4] = E;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------ k side
// One CTA per (key tile, head, sample); its key chunks [KH | Z | VH] stay
// resident.  Per query tile s:
//   ST(s):  S^T = Khat Qhat^T (M = keys; the Qhat chunks stream)
//   DPT(s): dP^T = Vhat dO^T into the same TMEM columns
//   GR(s):  with P^T and dS^T (fp16, K-major) written to shared memory by the
//           softmax warps: dK head += dS^T QH, dV head += P^T dO head,
//           dz2 += dS^T u hi + P^T dU, the B operands streamed again (the u hi
//           and dU rows as slices of 32 queries x every pair column, so that
//           each landed slot feeds two MMAs of the full width N = 64 nZ)
// issued as ST(0) DPT(0) [ST(s+1) GR(s) DPT(s+1)]....
constexpr int kKBarFull = 0, kKBarEmpty = 64, kKBarRes = 128, kKBarStFull = 136, kKBarStRead = 144,
              kKBarDpFull = 152, kKBarDpRead = 160, kKBarPdsFull = 168, kKBarGrDone = 176, kKBarQdFull = 184,
              kKBarQdEmpty = 200, kKBarDrain = 216;
constexpr int kKMisc = 256, kKOq = 512, kKQd = 1024, kKQdFloats = 9 * 128, kKTiles = 10240;
constexpr int kSliceGroupBytes = 32 * 128;   // one 32-row x 64-column fp16 box (128-byte swizzle)

__device__ __forceinline__ void zero_key_rows(const BwdArgs& a, int b, int h, int kt) {
  const Plan& p = a.p;
  const BwdPlan& bp = a.bp;
  const int bh = b * p.H + h;
  for (int e = threadIdx.x; e < kTile * bp.Kk; e += blockDim.x) {
    const int j = kt * kTile + e / bp.Kk;
    if (j < p.N) a.kres[((size_t)bh * p.N + kt * kTile) * bp.Kk + e] = 0.f;
  }
  for (int e = threadIdx.x; e < kTile * bp.RCz; e += blockDim.x) {
    const int j = kt * kTile + e / bp.RCz;
    if (j < p.N) a.dz2h[((size_t)bh * p.N + kt * kTile) * bp.RCz + e] = 0.f;
  }
}

__global__ void __launch_bounds__(256, 1)
bwd_k_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmKH,
             const __grid_constant__ CUtensorMap tmVH, const __grid_constant__ CUtensorMap tmZ,
             const __grid_constant__ CUtensorMap tmdO, const __grid_constant__ CUtensorMap tmQ32,
             const __grid_constant__ CUtensorMap tmdO32, const BwdArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const Plan& p = a.p;
  const BwdPlan& bp = a.bp;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int bh = b * p.H + h;
  const int N = p.N, nT = p.nT;
  if (a.flag[(size_t)b * nT + kt] == 0) {      // no valid key in this tile: zero gradients
    zero_key_rows(a, b, h, kt);
    return;
  }
  const int nKH = p.nKH, nZ = p.nZ, nVH = p.nVH, nqz = p.nqz;
  uint8_t* sK = smem;                                   // [KH | Z | VH] chunks of the key tile
  uint8_t* sP = sK + bp.k_nres * kChunkBytes;           // P^T  [128 keys x 128 queries] fp16, 2 chunks
  uint8_t* sD = sP + 2 * kChunkBytes;                   // dS^T
  uint8_t* sRing = sD + 2 * kChunkBytes;
  uint8_t* tail = sRing + bp.k_nst * kChunkBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(tail + kKBarFull);
  uint64_t* empty = reinterpret_cast<uint64_t*>(tail + kKBarEmpty);
  uint64_t* res_full = reinterpret_cast<uint64_t*>(tail + kKBarRes);
  uint64_t* st_full = reinterpret_cast<uint64_t*>(tail + kKBarStFull);
  uint64_t* st_read = reinterpret_cast<uint64_t*>(tail + kKBarStRead);
  uint64_t* dp_full = reinterpret_cast<uint64_t*>(tail + kKBarDpFull);
  uint64_t* dp_read = reinterpret_cast<uint64_t*>(tail + kKBarDpRead);
  uint64_t* pds_full = reinterpret_cast<uint64_t*>(tail + kKBarPdsFull);
  uint64_t* gr_done = reinterpret_cast<uint64_t*>(tail + kKBarGrDone);
  uint64_t* qd_full = reinterpret_cast<uint64_t*>(tail + kKBarQdFull);
  uint64_t* qd_empty = reinterpret_cast<uint64_t*>(tail + kKBarQdEmpty);
  uint64_t* drain = reinterpret_cast<uint64_t*>(tail + kKBarDrain);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tail + kKMisc);
  int* abort_flag = reinterpret_cast<int*>(tail + kKMisc + 4);
  int* ntiles = reinterpret_cast<int*>(tail + kKMisc + 8);
  float4* oqbuf = reinterpret_cast<float4*>(tail + kKOq);          // [2][4] query-group origins
  float* qdbuf = reinterpret_cast<float*>(tail + kKQd);            // [2][mb 4x128 | dd 4x128 | invl 128]
  uint16_t* tiles = reinterpret_cast<uint16_t*>(tail + kKTiles);

  if (threadIdx.x == 0) {
    for (int s = 0; s < bp.k_nst; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    mbar_init(res_full, 1);
    mbar_init(st_full, 1);
    mbar_init(st_read, 128);
    mbar_init(dp_full, 1);
    mbar_init(dp_read, 128);
    mbar_init(pds_full, 128);
    mbar_init(gr_done, 1);
    mbar_init(&qd_full[0], 64);
    mbar_init(&qd_full[1], 64);
    mbar_init(&qd_empty[0], 128);
    mbar_init(&qd_empty[1], 128);
    mbar_init(drain, 1);
    fence_mbar_init();
    *abort_flag = 0;
    int n = 0;
    const int* fl = a.flag + (size_t)b * nT;
    for (int t = 0; t < nT; ++t)
      if (fl[t]) tiles[n++] = (uint16_t)t;
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
  const int nq = *ntiles;
  const WaitCtx wc{abort_flag, a.status, a.timeout_ns};

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && nq > 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmKH);
      tma_prefetch_desc(&tmVH);
      tma_prefetch_desc(&tmZ);
      tma_prefetch_desc(&tmdO);
      tma_prefetch_desc(&tmQ32);
      tma_prefetch_desc(&tmdO32);
      mbar_arrive_expect_tx(res_full, (uint32_t)(bp.k_nres * kChunkBytes));
      for (int c = 0; c < nKH; ++c) tma_load_3d(sK + c * kChunkBytes, &tmKH, res_full, c * kChunk, kt * kTile, bh);
      for (int c = 0; c < nZ; ++c)
        tma_load_3d(sK + (nKH + c) * kChunkBytes, &tmZ, res_full, c * kChunk, kt * kTile, b);
      for (int c = 0; c < nVH; ++c)
        tma_load_3d(sK + (nKH + nZ + c) * kChunkBytes, &tmVH, res_full, c * kChunk, kt * kTile, bh);
      Ring rg{full, empty, sRing, bp.k_nst};
      bool ok = true;
      uint32_t issued = 0;
      auto push = [&](const CUtensorMap* tm, int c0, int qt) {
        if (!ok) return;
        if (!mbar_wait(&empty[rg.st], rg.ph ^ 1u, wc, 41)) { ok = false; return; }
        mbar_arrive_expect_tx(&full[rg.st], kChunkBytes);
        tma_load_3d(rg.slot(), tm, &full[rg.st], c0, qt * kTile, bh);
        ++issued;
        rg.next();
      };
      auto push_st = [&](int qt) {
        for (int c = 0; c < nZ; ++c)
          for (int qz = 0; qz < nqz; ++qz) push(&tmQ, (nKH + qz * nZ + c) * kChunk, qt);
        for (int c = 0; c < nKH; ++c) push(&tmQ, c * kChunk, qt);
      };
      auto push_dp = [&](int qt) {
        for (int c = 0; c < bp.nOc; ++c) push(&tmdO, c * kChunk, qt);
      };
      // one slot = 32 queries x the nZ 64-column groups from column col0, one
      // 32-row box per group, 4 KB apart (a K slice of an N = 64 nZ operand)
      auto push_slices = [&](const CUtensorMap* tm, int col0, int qt) {
        for (int sl = 0; sl < kTile / 32; ++sl) {
          if (!ok) return;
          if (!mbar_wait(&empty[rg.st], rg.ph ^ 1u, wc, 41)) { ok = false; return; }
          mbar_arrive_expect_tx(&full[rg.st], (uint32_t)(nZ * kSliceGroupBytes));
          for (int c = 0; c < nZ; ++c)
            tma_load_3d(rg.slot() + c * kSliceGroupBytes, tm, &full[rg.st], col0 + c * kChunk, qt * kTile + sl * 32,
                        bh);
          ++issued;
          rg.next();
        }
      };
      // gradient products: QH, dO head, then the u hi and dU slices (the dz2
      // product uses u hi only: the lo half is 2^-12 of u, far below the
      // gradient tolerance; the logits above are recomputed with both halves)
      auto push_gr = [&](int qt) {
        for (int c = 0; c < nKH; ++c) push(&tmQ, c * kChunk, qt);
        for (int c = 0; c < nVH; ++c) push(&tmdO, c * kChunk, qt);
        push_slices(&tmQ32, nKH * kChunk, qt);
        push_slices(&tmdO32, nVH * kChunk, qt);
      };
      push_st(tiles[0]);
      push_dp(tiles[0]);
      for (int s = 0; s < nq && ok; ++s) {
        if (s + 1 < nq) push_st(tiles[s + 1]);
        push_gr(tiles[s]);
        if (s + 1 < nq) push_dp(tiles[s + 1]);
      }
      if (*abort_flag) {
        bwd_drain_wait(res_full, 0, a.timeout_ns);
        const uint32_t last = issued < (uint32_t)bp.k_nst ? issued : (uint32_t)bp.k_nst;
        for (uint32_t k = 0; k < last; ++k) {
          const uint32_t n = issued - 1 - k;
          bwd_drain_wait(&full[n % bp.k_nst], (n / bp.k_nst) & 1u, a.timeout_ns);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && nq > 0) {
      bool ok = mbar_wait(res_full, 0, wc, 42);
      tc_fence_after();
      Ring rg{full, empty, sRing, bp.k_nst};
      const uint32_t idS = idesc_f16(128, 128, 0, 0);
      const uint32_t sKa = smem_u32(sK), sPa = smem_u32(sP), sDa = smem_u32(sD), ringa = smem_u32(sRing);
      auto take = [&](int site) -> int {
        if (!mbar_wait(&full[rg.st], rg.ph, wc, site)) return -1;
        tc_fence_after();
        const int st = rg.st;
        rg.next();
        return st;
      };
      // A = P^T or dS^T: K-major [128 keys x 128 queries]; K step kk = 16 queries
      auto adesc = [&](uint32_t base, int kk) -> uint64_t {
        return desc_kmajor_sw128(base + (uint32_t)(kk >> 2) * kChunkBytes + (uint32_t)(kk & 3) * 32);
      };
      auto mma_st = [&]() -> bool {
        bool first = true;
        for (int c = 0; c < nZ; ++c) {
          const uint32_t az = sKa + (nKH + c) * kChunkBytes;
          for (int qz = 0; qz < nqz; ++qz) {
            const int sl = take(43);
            if (sl < 0) return false;
            const uint32_t bq = ringa + sl * kChunkBytes;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_ss(tmem, desc_kmajor_sw128(az + kk * 32), desc_kmajor_sw128(bq + kk * 32), idS,
                     (!first || kk > 0) ? 1u : 0u);
            first = false;
            tc_commit(&empty[sl]);
          }
        }
        for (int c = 0; c < nKH; ++c) {
          const int sl = take(43);
          if (sl < 0) return false;
          const uint32_t bq = ringa + sl * kChunkBytes, ak = sKa + c * kChunkBytes;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ss(tmem, desc_kmajor_sw128(ak + kk * 32), desc_kmajor_sw128(bq + kk * 32), idS,
                   (!first || kk > 0) ? 1u : 0u);
          first = false;
          tc_commit(&empty[sl]);
        }
        tc_commit(st_full);
        return true;
      };
      auto mma_dp = [&]() -> bool {
        for (int c = 0; c < bp.nOc; ++c) {
          const int sl = take(44);
          if (sl < 0) return false;
          const uint32_t bo = ringa + sl * kChunkBytes;
          const uint32_t av = c < nVH ? sKa + (nKH + nZ + c) * kChunkBytes : sKa + (nKH + c - nVH) * kChunkBytes;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ss(tmem, desc_kmajor_sw128(av + kk * 32), desc_kmajor_sw128(bo + kk * 32), idS, (c | kk) != 0);
          tc_commit(&empty[sl]);
        }
        tc_commit(dp_full);
        return true;
      };
      // `nch` chunks into consecutive 64-column blocks from `dcol`: chunks in
      // consecutive ring slots form one MMA of N = 64 x run (MN-major B, groups
      // one slot apart), up to 4 chunks
      auto gr_run = [&](uint32_t dcol, uint32_t abase, int nch, bool acc0, int site) -> bool {
        for (int c = 0; c < nch;) {
          int run = nch - c;
          if (run > 4) run = 4;
          if (run > rg.nst - rg.st) run = rg.nst - rg.st;
          for (int u = 0; u < run; ++u)
            if (!mbar_wait(&full[rg.st + u], rg.ph, wc, site)) return false;
          tc_fence_after();
          const uint32_t bq = ringa + rg.st * kChunkBytes;
          const uint32_t idR = idesc_f16(128, 64 * run, 0, 1);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ss(dcol + (uint32_t)(c * kChunk), adesc(abase, kk), desc_mnmajor_sw128(bq + kk * 2048, kChunkBytes),
                   idR, (acc0 || kk > 0) ? 1u : 0u);
          for (int u = 0; u < run; ++u) tc_commit(&empty[rg.st + u]);
          rg.st += run;
          if (rg.st == rg.nst) { rg.st = 0; rg.ph ^= 1u; }
          c += run;
        }
        return true;
      };
      // dz2 += dS^T u hi + P^T dU: per slot of 32 queries, two K steps of one
      // MMA over all 64 nZ columns (MN-major B, column groups 4 KB apart)
      const uint32_t idZ = idesc_f16(128, 64 * nZ, 0, 1);
      auto mma_gr = [&](int s) -> bool {
        const bool acc0 = s > 0;
        if (!gr_run(tmem + (uint32_t)bp.tmDK, sDa, nKH, acc0, 45)) return false;
        if (!gr_run(tmem + (uint32_t)bp.tmDV, sPa, nVH, acc0, 46)) return false;
        for (int part = 0; part < 2; ++part) {
          const uint32_t abase = part == 0 ? sDa : sPa;
          for (int sl = 0; sl < kTile / 32; ++sl) {
            const int st = take(part == 0 ? 47 : 48);
            if (st < 0) return false;
            const uint32_t bq = ringa + st * kChunkBytes;
#pragma unroll
            for (int kk = 0; kk < 2; ++kk)
              mma_ss(tmem + (uint32_t)bp.tmDZ, adesc(abase, 2 * sl + kk),
                     desc_mnmajor_sw128(bq + kk * 2048, kSliceGroupBytes), idZ,
                     (part > 0 || acc0 || sl > 0 || kk > 0) ? 1u : 0u);
            tc_commit(&empty[st]);
          }
        }
        tc_commit(gr_done);
        return true;
      };
      if (ok) ok = mma_st();
      if (ok) ok = mbar_wait(st_read, 0, wc, 49);
      if (ok) { tc_fence_after(); ok = mma_dp(); }
      for (int s = 0; ok && s < nq; ++s) {
        if (s + 1 < nq) {
          if (!mbar_wait(dp_read, s & 1, wc, 50)) break;
          tc_fence_after();
          if (!mma_st()) break;
        }
        if (!mbar_wait(pds_full, s & 1, wc, 51)) break;
        tc_fence_after();
        if (!mma_gr(s)) break;
        if (s + 1 < nq) {
          if (!mbar_wait(st_read, (s + 1) & 1, wc, 52)) break;
          tc_fence_after();
          if (!mma_dp()) break;
        }
      }
      tc_commit(drain);
      bwd_drain_wait(drain, 0, a.timeout_ns);
    }
  } else if (warp == 2 || warp == 3) {
    // ------------------------------------------------------------ per-query terms
    // for query i and key group t of this tile: mb = M_i - rc(i,t) log2e with
    // rc = -g (P |D|^2 + 2 D . sum_p a'_p), D = o_{group(i)} - o_t; dd = sG_i . o_t - D_i;
    // invl = 1/l_i (0 for a query without a permitted key)
    const int tt = threadIdx.x - 64;
    const float g = point_weight(bwd_raw(a, h), p.P);
    float4 okt[4];
#pragma unroll
    for (int t = 0; t < 4; ++t) okt[t] = a.orig[(size_t)b * p.nG + kt * 4 + t];
    for (int s = 0; s < nq; ++s) {
      const int kb = s & 1;
      const bool okw = mbar_wait(&qd_empty[kb], ((s >> 1) & 1) ^ 1, wc, 53);
      if (!__all_sync(0xffffffffu, okw)) break;
      const int qt = tiles[s];
      float* qd = qdbuf + kb * kKQdFloats;
      if (tt < 4) oqbuf[kb * 4 + tt] = a.orig[(size_t)b * p.nG + qt * 4 + tt];
      for (int il = tt; il < kTile; il += 64) {
        const int i = qt * kTile + il;
        const bool in = i < N;
        const bool valid = in && a.mask[(size_t)b * N + i] != 0;
        const float2 stt = in ? a.stats[(size_t)bh * N + i] : make_float2(0.f, 0.f);
        const float invl = (valid && stt.y > 0.f) ? 1.f / stt.y : 0.f;
        const float4 qv = in ? a.qvec[(size_t)bh * N + i] : make_float4(0.f, 0.f, 0.f, 0.f);
        const float4 dvv = in ? a.dvec[(size_t)bh * N + i] : make_float4(0.f, 0.f, 0.f, 0.f);
        const float4 og = a.orig[(size_t)b * p.nG + qt * 4 + (il >> 5)];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const float dx = og.x - okt[t].x, dy = og.y - okt[t].y, dz = og.z - okt[t].z;
          const float rc = -g * ((float)p.P * (dx * dx + dy * dy + dz * dz) + 2.f * (dx * qv.x + dy * qv.y + dz * qv.z));
          qd[t * kTile + il] = invl > 0.f ? stt.x - rc * kLog2e : 0.f;
          qd[512 + t * kTile + il] = dvv.y * okt[t].x + dvv.z * okt[t].y + dvv.w * okt[t].z - dvv.x;
        }
        qd[1024 + il] = invl;
      }
      mbar_arrive(&qd_full[kb]);
    }
  } else {
    // ------------------------------------------------------------ softmax warps
    // thread = key j = TMEM lane; a row of S^T holds the 128 queries of the tile
    const int wq = warp - 4;
    const int r = wq * 32 + lane;
    const int j = kt * kTile + r;
    const bool jin = j < N;
    const float4 kv = jin ? a.kvec[(size_t)bh * N + j] : make_float4(-INFINITY, 0.f, 0.f, 0.f);
    const float4 okj = a.orig[(size_t)b * p.nG + kt * 4 + wq];
    const float g = point_weight(bwd_raw(a, h), p.P);
    const uint32_t trow = tmem + ((uint32_t)(wq * 32) << 16);
    float cs = 0.f, Vx = 0.f, Vy = 0.f, Vz = 0.f;
    bool ok = true;
    for (int s = 0; s < nq; ++s) {
      const int qt = tiles[s];
      const int kb = s & 1;
      ok = mbar_wait(st_full, s & 1, wc, 54);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      tc_fence_after();
      uint32_t sv[4][32];
      tmem_ld32(trow + 0, sv[0]);
      tmem_ld32(trow + 32, sv[1]);
      tmem_ld32(trow + 64, sv[2]);
      tmem_ld32(trow + 96, sv[3]);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(st_read);
      ok = mbar_wait(&qd_full[kb], (s >> 1) & 1, wc, 55);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      const float* qd = qdbuf + kb * kKQdFloats;
      const float* mbw = qd + wq * kTile;
      const float* ddw = qd + 512 + wq * kTile;
      const float* ilw = qd + 1024;
      float4 oq[4];
      float ktm[4];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        oq[t] = oqbuf[kb * 4 + t];
        const float dx = oq[t].x - okj.x, dy = oq[t].y - okj.y, dz = oq[t].z - okj.z;
        ktm[t] = kv.x + 2.f * g * (dx * kv.y + dy * kv.z + dz * kv.w);
      }
      // a forbidden pair gets the logit -inf in a pass of its own, so that the
      // loop below has no branch (an absent key has kterm -inf already)
      if (a.pair_mask != nullptr) {
        const uint8_t* pmcol = a.pair_mask + (size_t)b * N * N + (jin ? j : 0);
        const uint4 b4 = pair_bits128(pmcol, (size_t)N, qt * kTile, N);
        const uint32_t bw[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
        for (int t = 0; t < 4; ++t)
#pragma unroll
          for (int e = 0; e < 32; ++e)
            sv[t][e] = ((bw[t] >> e) & 1u) ? sv[t][e] : __float_as_uint(-INFINITY);
      }
      uint32_t pk[2][32];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          float pv[2];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int il = t * 32 + e + u;
            const float il_inv = ilw[il];
            const float x = __uint_as_float(sv[t][e + u]) + ktm[t];
            pv[u] = il_inv > 0.f ? ex2_approx(fmaf(x, kLog2e, -mbw[il])) * il_inv : 0.f;
          }
          pk[t >> 1][(t & 1) * 16 + e / 2] = pack_half2(pv[0], pv[1]);
        }
      }
      ok = mbar_wait(dp_full, s & 1, wc, 56);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      tc_fence_after();
      tmem_ld32(trow + 0, sv[0]);
      tmem_ld32(trow + 32, sv[1]);
      tmem_ld32(trow + 64, sv[2]);
      tmem_ld32(trow + 96, sv[3]);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(dp_read);
      uint32_t dk[2][32];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        float cst = 0.f;
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const int w = (t & 1) * 16 + e / 2;
          const float2 pp = __half22float2(*reinterpret_cast<const __half2*>(&pk[t >> 1][w]));
          const int il = t * 32 + e;
          const float d0 = pp.x * (__uint_as_float(sv[t][e]) + ddw[il]);
          const float d1 = pp.y * (__uint_as_float(sv[t][e + 1]) + ddw[il + 1]);
          const __half2 hd = __floats2half2_rn(d0, d1);
          const float2 fd = __half22float2(hd);
          cst += fd.x + fd.y;
          dk[t >> 1][w] = *reinterpret_cast<const uint32_t*>(&hd);
        }
        cs += cst;
        Vx = fmaf(cst, oq[t].x, Vx);
        Vy = fmaf(cst, oq[t].y, Vy);
        Vz = fmaf(cst, oq[t].z, Vz);
      }
      mbar_arrive(&qd_empty[kb]);
      if (s > 0) {
        ok = mbar_wait(gr_done, (s - 1) & 1, wc, 57);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        tc_fence_after();
      }
      // row r of P^T and dS^T, 128-byte swizzle: 16-byte unit u of the row sits
      // at unit u ^ (r & 7)
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint8_t* rp = sP + c * kChunkBytes + r * 128;
        uint8_t* rd = sD + c * kChunkBytes + r * 128;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int pu = (u ^ (r & 7)) << 4;
          *reinterpret_cast<uint4*>(rp + pu) = make_uint4(pk[c][4 * u], pk[c][4 * u + 1], pk[c][4 * u + 2], pk[c][4 * u + 3]);
          *reinterpret_cast<uint4*>(rd + pu) = make_uint4(dk[c][4 * u], dk[c][4 * u + 1], dk[c][4 * u + 2], dk[c][4 * u + 3]);
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(pds_full);
    }
    if (ok && nq > 0) {
      ok = mbar_wait(gr_done, (nq - 1) & 1, wc, 58);
      ok = __all_sync(0xffffffffu, ok);
      tc_fence_after();
    }
    // tcgen05.ld is warp-collective: every lane loads, only keys in range store
    const bool aborted = __any_sync(0xffffffffu, *abort_flag != 0);
    const bool wr = jin && !aborted;
    float* kr = a.kres + ((size_t)bh * N + (jin ? j : 0)) * bp.Kk;
    float* dzr = a.dz2h + ((size_t)bh * N + (jin ? j : 0)) * bp.RCz;
    const int D = p.D, P3 = 3 * p.P, Dv = p.Dv;
    const int ofs_cs = D + P3, ofs_dv = D + P3 + 4, ofs_dg = D + P3 + 4 + Dv;
    float ylo[3 * kMaxPts];
#pragma unroll 1
    for (int x = 0; x < P3; ++x) ylo[x] = 0.f;
    // dK head: [sum dS q/sqrt(3D) | 2g a' hi | 2g a' hi | 2g a' lo]
    for (int c0 = 0; c0 < 64 * nKH; c0 += 32) {
      uint32_t o[32];
      tmem_ld32(trow + (uint32_t)(bp.tmDK + c0), o);
      tmem_ld_wait();
      if (wr) {
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int c = c0 + e;
          const float v = __uint_as_float(o[e]);
          if (c < D) kr[c] = v;
          else if (c >= p.D8 && c < p.D8 + P3) kr[D + c - p.D8] = v;
          else if (c >= p.D8 + 2 * p.P38 && c < p.D8 + 2 * p.P38 + P3) ylo[c - p.D8 - 2 * p.P38] = v;
        }
      }
    }
    // dV head: [sum P d o_scalar | sum P dG | (copy) | 0]
    for (int c0 = 0; c0 < 64 * nVH; c0 += 32) {
      uint32_t o[32];
      tmem_ld32(trow + (uint32_t)(bp.tmDV + c0), o);
      tmem_ld_wait();
      if (wr) {
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int c = c0 + e;
          const float v = __uint_as_float(o[e]);
          if (c < Dv) kr[ofs_dv + c] = v;
          else if (c >= p.Dv8 && c < p.Dv8 + 3 * p.Q) kr[ofs_dg + c - p.Dv8] = v;
        }
      }
    }
    for (int c0 = 0; c0 < 64 * nZ; c0 += 32) {
      uint32_t o[32];
      tmem_ld32(trow + (uint32_t)(bp.tmDZ + c0), o);
      tmem_ld_wait();
      if (wr) {
#pragma unroll
        for (int e = 0; e < 32; ++e)
          if (c0 + e < bp.RCz) dzr[c0 + e] = __uint_as_float(o[e]);
      }
    }
    if (wr) {
      for (int x = 0; x < P3; ++x) kr[D + x] += ylo[x];
      kr[ofs_cs] = cs;
      kr[ofs_cs + 1] = Vx;
      kr[ofs_cs + 2] = Vy;
      kr[ofs_cs + 3] = Vz;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------ chain
// One CTA per kChainRes residues.  Items (residue, head): the scalar
// gradients, the points through the frames (a = R x + t: dx = R^T da,
// dR += da (x) x, dt += da) and this row's part of the distance-weight
// gradient; then per residue the frame gradients summed over heads in head
// order, and per (residue, pair column) the factor gradients
//   dz1[r,c] = (from the prep) + sum_h du_h[r,c] Wb[c,h] / sqrt(3),  dz2 = sum_h dz2_h,
// and the CTA's partial sums of dWb and of the distance-weight gradient.
__global__ void __launch_bounds__(256) bwd_chain_kernel(const BwdArgs a) {
  const Plan& p = a.p;
  const BwdPlan& bp = a.bp;
  extern __shared__ float csm[];
  const int H = p.H, P = p.P, Q = p.Q, D = p.D, Dv = p.Dv, RCz = bp.RCz, Cz = p.Cz, N = p.N;
  const int total = p.B * N;
  const int bi0 = blockIdx.x * kChainRes;
  const int nres = min(kChainRes, total - bi0);
  const int tid = threadIdx.x;
  float* red = csm;                                  // [kChainRes * H][12]
  float* gam = red + kChainRes * H * 12;             // [kChainRes * H]
  float* frm = gam + kChainRes * H;                  // [kChainRes][16]: R, t, origin
  for (int r = tid; r < nres; r += blockDim.x) {
    const int bi = bi0 + r, b = bi / N, i = bi - b * N;
    float* f = frm + r * 16;
    for (int e = 0; e < 9; ++e) f[e] = ldi(a.rot, (size_t)bi * 9 + e, a.p.in_f32);
    for (int e = 0; e < 3; ++e) f[9 + e] = ldi(a.trans, (size_t)bi * 3 + e, a.p.in_f32);
    const float4 o = a.orig[(size_t)b * p.nG + i / kGroup];
    f[12] = o.x; f[13] = o.y; f[14] = o.z;
  }
  __syncthreads();
  const float s3D = rsqrtf(3.f * (float)D);
  for (int it = tid; it < nres * H; it += blockDim.x) {
    const int r = it / H, h = it - r * H;
    const int bi = bi0 + r, b = bi / N, i = bi - b * N;
    const size_t idx = ((size_t)b * H + h) * N + i;
    const size_t bih = (size_t)bi * H + h;
    const float* f = frm + r * 16;
    const float* Rm = f;
    const float t[3] = {f[9], f[10], f[11]};
    const float o[3] = {f[12], f[13], f[14]};
    const float g = point_weight(bwd_raw(a, h), P);
    const float g2 = 2.f * g;
    const float* qr = a.qres + idx * bp.Kr;
    const float* kr = a.kres + idx * bp.Kk;
    const float rs = qr[D + 3 * P], E = qr[D + 3 * P + 4];
    const float W[3] = {qr[D + 3 * P + 1], qr[D + 3 * P + 2], qr[D + 3 * P + 3]};
    const float cs = kr[D + 3 * P];
    const float V[3] = {kr[D + 3 * P + 1], kr[D + 3 * P + 2], kr[D + 3 * P + 3]};
    for (int d = 0; d < D; ++d) {
      a.g.q[bih * D + d] = qr[d] * s3D;
      a.g.k[bih * D + d] = kr[d];
    }
    for (int d = 0; d < Dv; ++d) a.g.v[bih * Dv + d] = kr[D + 3 * P + 4 + d];
    float dR[9], dt[3];
#pragma unroll
    for (int e = 0; e < 9; ++e) dR[e] = 0.f;
    dt[0] = dt[1] = dt[2] = 0.f;
    float gm = 0.f;
    auto frame_back = [&](const float (&x)[3], const float (&dg)[3], float* out) {
      // point x (local) -> R x + t: dx = R^T dg, dR += dg (x) x, dt += dg
#pragma unroll
      for (int c = 0; c < 3; ++c) out[c] = Rm[c] * dg[0] + Rm[3 + c] * dg[1] + Rm[6 + c] * dg[2];
#pragma unroll
      for (int rr = 0; rr < 3; ++rr) {
#pragma unroll
        for (int c = 0; c < 3; ++c) dR[3 * rr + c] += dg[rr] * x[c];
        dt[rr] += dg[rr];
      }
    };
    for (int pp = 0; pp < P; ++pp) {
      float xq[3], xk[3], ap[3], bpp[3], da[3], db[3];
      for (int c = 0; c < 3; ++c) {
        xq[c] = ldi(a.q_pts, (bih * P + pp) * 3 + c, a.p.in_f32);
        xk[c] = ldi(a.k_pts, (bih * P + pp) * 3 + c, a.p.in_f32);
      }
#pragma unroll
      for (int rr = 0; rr < 3; ++rr) {
        ap[rr] = Rm[3 * rr] * xq[0] + Rm[3 * rr + 1] * xq[1] + Rm[3 * rr + 2] * xq[2] + t[rr] - o[rr];
        bpp[rr] = Rm[3 * rr] * xk[0] + Rm[3 * rr + 1] * xk[1] + Rm[3 * rr + 2] * xk[2] + t[rr] - o[rr];
      }
#pragma unroll
      for (int c = 0; c < 3; ++c) {
        const float X = qr[D + 3 * pp + c];
        da[c] = g2 * ((X - rs * ap[c]) + (W[c] - rs * o[c]));
        db[c] = kr[D + 3 * pp + c] + g2 * (V[c] - cs * o[c]) - g2 * cs * bpp[c];
        gm += rs * ap[c] * ap[c] - 2.f * ap[c] * X;
      }
      frame_back(xq, da, a.g.q_pts + (bih * P + pp) * 3);
      frame_back(xk, db, a.g.k_pts + (bih * P + pp) * 3);
    }
    for (int q = 0; q < Q; ++q) {
      float xv[3], dg[3];
      for (int c = 0; c < 3; ++c) {
        xv[c] = ldi(a.v_pts, (bih * Q + q) * 3 + c, a.p.in_f32);
        dg[c] = kr[D + 3 * P + 4 + Dv + 3 * q + c];
      }
      frame_back(xv, dg, a.g.v_pts + (bih * Q + q) * 3);
    }
    if (g > 0.f) gm -= E / g;
    gam[it] = -gm;
#pragma unroll
    for (int e = 0; e < 9; ++e) red[it * 12 + e] = dR[e];
    red[it * 12 + 9] = dt[0];
    red[it * 12 + 10] = dt[1];
    red[it * 12 + 11] = dt[2];
  }
  __syncthreads();
  for (int e = tid; e < nres * 12; e += blockDim.x) {
    const int r = e / 12, k = e - r * 12;
    const int bi = bi0 + r;
    float s = a.rloc[(size_t)bi * 12 + k];
    for (int h = 0; h < H; ++h) s += red[(r * H + h) * 12 + k];
    if (k < 9) a.g.rot[(size_t)bi * 9 + k] = s;
    else a.g.trans[(size_t)bi * 3 + k - 9] = s;
  }
  for (int h = tid; h < H; h += blockDim.x) {
    float s = 0.f;
    for (int r = 0; r < nres; ++r) s += gam[r * H + h];
    a.gpart[(size_t)blockIdx.x * H + h] = s;
  }
  for (int e = tid; e < nres * RCz; e += blockDim.x) {
    const int r = e / RCz, rc = e - r * RCz, c = rc % Cz;
    const int bi = bi0 + r, b = bi / N, i = bi - b * N;
    float s1 = a.dz1u[(size_t)bi * RCz + rc], s2 = 0.f;
    for (int h = 0; h < H; ++h) {
      const size_t idx = ((size_t)b * H + h) * N + i;
      s1 = fmaf(a.du[idx * RCz + rc], ldi(a.Wb, (size_t)c * H + h, a.p.in_f32) * kInvSqrt3, s1);
      s2 += a.dz2h[idx * RCz + rc];
    }
    a.g.z1[(size_t)bi * RCz + rc] = s1;
    a.g.z2[(size_t)bi * RCz + rc] = s2;
  }
  // dWb partials: consecutive threads take consecutive channels c (coalesced
  // du and z1 rows); the result lands at [c][h]
  for (int e = tid; e < Cz * H; e += blockDim.x) {
    const int h = e / Cz, c = e - h * Cz;
    float s = 0.f;
    for (int r = 0; r < nres; ++r) {
      const int bi = bi0 + r, b = bi / N, i = bi - b * N;
      const size_t idx = ((size_t)b * H + h) * N + i;
      for (int rr = 0; rr < p.R; ++rr)
        s = fmaf(a.du[idx * RCz + rr * Cz + c], ldi(a.z1, (size_t)bi * RCz + rr * Cz + c, a.p.in_f32), s);
    }
    a.wbpart[(size_t)blockIdx.x * Cz * H + (size_t)c * H + h] = s * kInvSqrt3;
  }
}

// dWb[c, h] and d point_w_raw[h]: the chain CTAs' partial sums, added in a
// fixed order (deterministic): 32 outputs per CTA, one per lane; warp g of the
// 8 sums the partials k = g, g + 8, ... in four interleaved accumulators (the
// loads in flight together), and lane e of warp 0 adds the 8 warps' sums in
// order.  d raw = d g * 1/2 sigmoid(raw) sqrt(2/(27P)) (softplus' = sigmoid).
constexpr int kFinalOut = 32;
__global__ void __launch_bounds__(256) bwd_final_kernel(const BwdArgs a) {
  __shared__ float red[8][kFinalOut + 1];
  const Plan& p = a.p;
  const int CH = p.Cz * p.H, nout = CH + p.H, nk = a.bp.nchain;
  const int lane = threadIdx.x & 31, grp = threadIdx.x >> 5;
  const int e = blockIdx.x * kFinalOut + lane;
  float acc0 = 0.f, acc1 = 0.f, acc2 = 0.f, acc3 = 0.f;
  if (e < nout) {
    const float* src = e < CH ? a.wbpart + e : a.gpart + (e - CH);
    const size_t stride = e < CH ? (size_t)CH : (size_t)p.H;
    for (int k = grp; k < nk; k += 32) {
      acc0 += src[(size_t)k * stride];
      if (k + 8 < nk) acc1 += src[(size_t)(k + 8) * stride];
      if (k + 16 < nk) acc2 += src[(size_t)(k + 16) * stride];
      if (k + 24 < nk) acc3 += src[(size_t)(k + 24) * stride];
    }
  }
  red[grp][lane] = (acc0 + acc1) + (acc2 + acc3);
  __syncthreads();
  if (grp == 0 && e < nout) {
    float s = 0.f;
#pragma unroll
    for (int g = 0; g < 8; ++g) s += red[g][lane];
    if (e < CH) {
      a.g.Wb[e] = s;
    } else {
      const int h = e - CH;
      const float raw = bwd_raw(a, h);
      const float sig = 1.f / (1.f + expf(-raw));
      a.g.raw[h] = s * 0.5f * sig * sqrtf(2.f / (27.f * (float)p.P));
    }
  }
}

}  // namespace

// The prep's form: one CTA of 8 warps per residue while the residues are
// fewer than kPrepWarpMin (more threads per residue), else one warp per residue
// and up to 8 residues per CTA (each warp's dG rows within 48 KB).
constexpr int kPrepWarpMin = 8192;
bool bwd_prep_cta(const Plan& p) { return p.B * p.N < kPrepWarpMin; }
int bwd_prep_wpc(const Plan& p) {
  if (bwd_prep_cta(p)) return 1;
  const size_t per = (size_t)rup(p.H * 3 * p.Q, 4) * 4;
  const size_t w = per > 0 ? 49152 / per : 8;
  return w >= 8 ? 8 : (w < 1 ? 1 : (int)w);
}
size_t bwd_prep_smem(const Plan& p) {
  return ((size_t)bwd_prep_wpc(p) * rup(p.H * 3 * p.Q, 4) + (bwd_prep_cta(p) ? 8 * 12 : 0)) * 4;
}
size_t bwd_chain_smem(const Plan& p) {
  return ((size_t)kChainRes * p.H * 13 + kChainRes * 16) * 4;
}

cudaError_t launch_backward(const Plan& p, const BwdPlan& bp, const Inputs& in, const Work& w, const BwdIO& io,
                            const CUtensorMap& tmQ, const CUtensorMap& tmKH, const CUtensorMap& tmVH,
                            const CUtensorMap& tmZ, const BwdMaps& bm, const DeviceCtl& ctl, cudaStream_t s,
                            StageMark mark, void* mark_ctx) {
  auto stage = [&](int k) {
    if (mark != nullptr) mark(mark_ctx, k);
  };
  BwdArgs a;
  a.p = p;
  a.bp = bp;
  a.q_pts = in.q_pts; a.k_pts = in.k_pts; a.v_pts = in.v_pts; a.rot = in.rot; a.trans = in.trans;
  a.z1 = in.z1; a.Wb = in.Wb; a.raw = in.raw; a.w_out = in.w_out;
  a.mask = in.mask; a.pair_mask = in.pair_mask; a.eps = in.eps;
  a.d_update = io.d_update; a.d_local = io.d_local;
  a.kvec = w.kvec; a.qvec = w.qvec; a.orig = w.orig; a.flag = w.flag; a.stats = w.stats; a.rowflag = w.rowflag;
  uint8_t* ws = io.ws;
  a.osave = reinterpret_cast<float*>(ws + bp.off_osave);
  a.dfeat = reinterpret_cast<float*>(ws + bp.off_dfeat);
  a.fhi = reinterpret_cast<__nv_bfloat16*>(ws + bp.off_fhi);
  a.flo = reinterpret_cast<__nv_bfloat16*>(ws + bp.off_flo);
  a.dO = reinterpret_cast<__half*>(ws + bp.off_dO);
  a.dvec = reinterpret_cast<float4*>(ws + bp.off_dvec);
  a.rloc = reinterpret_cast<float*>(ws + bp.off_rloc);
  a.dz1u = reinterpret_cast<float*>(ws + bp.off_dz1u);
  a.qres = reinterpret_cast<float*>(ws + bp.off_qres);
  a.du = reinterpret_cast<float*>(ws + bp.off_du);
  a.kres = reinterpret_cast<float*>(ws + bp.off_kres);
  a.dz2h = reinterpret_cast<float*>(ws + bp.off_dz2h);
  a.dwpart = reinterpret_cast<float*>(ws + bp.off_dwpart);
  a.wbpart = reinterpret_cast<float*>(ws + bp.off_wbpart);
  a.gpart = reinterpret_cast<float*>(ws + bp.off_gpart);
  a.g = io.g;
  a.status = ctl.status;
  a.timeout_ns = ctl.timeout_ns;
  const int BN = p.B * p.N;
  cudaError_t e;
  stage(1);
  // dfeat = d_update w_out^T: d_update and w_out as bfloat16 hi / lo rows of Coutp
  // columns; w_out given in bfloat16 is exact in its hi part
  __nv_bfloat16* duhi = reinterpret_cast<__nv_bfloat16*>(ws + bp.off_duhi);
  __nv_bfloat16* dulo = reinterpret_cast<__nv_bfloat16*>(ws + bp.off_dulo);
  if ((e = launch_bsplit(io.d_update, 1, duhi, dulo, BN, p.Cout, bp.Coutp, s)) != cudaSuccess) return e;
  if ((e = launch_bsplit(in.w_out, p.in_f32, reinterpret_cast<__nv_bfloat16*>(ws + bp.off_whi),
                         reinterpret_cast<__nv_bfloat16*>(ws + bp.off_wlo), p.F, p.Cout, bp.Coutp, s)) != cudaSuccess)
    return e;
  {
    BGemm g{};
    g.A[0] = bm.duA[0]; g.A[1] = bm.duA[1]; g.B[0] = bm.w[0]; g.B[1] = bm.w[1];
    g.a_mn = 0; g.b_mn = 0;
    g.M = BN; g.N = p.F; g.K = bp.Coutp;
    g.nparts = p.in_f32 ? 3 : 2;
    g.pa[0] = 0; g.pb[0] = 0;      // d hi  w hi
    g.pa[1] = 1; g.pb[1] = 0;      // d lo  w hi
    g.pa[2] = 0; g.pb[2] = 1;      // d hi  w lo (float32 w_out)
    g.splits = 1;
    g.C = a.dfeat; g.ldc = p.F; g.zstride = 0;
    g.status = ctl.status; g.timeout_ns = ctl.timeout_ns;
    if ((e = launch_bgemm(g, s)) != cudaSuccess) return e;
  }
  const int wpc = bwd_prep_wpc(p);
  const size_t psm = bwd_prep_smem(p);
  if (bwd_prep_cta(p)) {
    if (psm > 48 * 1024 &&
        (e = cudaFuncSetAttribute(bwd_prep_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)psm)) !=
            cudaSuccess)
      return e;
    bwd_prep_kernel<8><<<BN, 256, psm, s>>>(a, 1);
  } else {
    bwd_prep_kernel<1><<<cdiv(BN, wpc), 32 * wpc, psm, s>>>(a, wpc);
  }
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if ((e = allow_max_smem(reinterpret_cast<const void*>(bwd_q_kernel))) != cudaSuccess) return e;
  stage(2);
  bwd_q_kernel<<<dim3(p.nT, p.H, p.B), 256, bp.q_smem, s>>>(tmQ, tmKH, tmVH, tmZ, *bm.dO, a);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if ((e = allow_max_smem(reinterpret_cast<const void*>(bwd_k_kernel))) != cudaSuccess) return e;
  stage(3);
  bwd_k_kernel<<<dim3(p.nT, p.H, p.B), 256, bp.k_smem, s>>>(tmQ, tmKH, tmVH, tmZ, *bm.dO, *bm.Q32, *bm.dO32, a);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  stage(4);
  const size_t csm = bwd_chain_smem(p);
  if (csm > 48 * 1024) {
    if ((e = cudaFuncSetAttribute(bwd_chain_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)csm)) != cudaSuccess)
      return e;
  }
  bwd_chain_kernel<<<bp.nchain, 256, csm, s>>>(a);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  {
    // [dw_out | db_out] partials = features^T d_update over row splits (the
    // feature rows carry a 1 in column F, so row F of the result is db_out)
    BGemm g{};
    g.A[0] = bm.f[0]; g.A[1] = bm.f[1]; g.B[0] = bm.duB[0]; g.B[1] = bm.duB[1];
    g.a_mn = 1; g.b_mn = 1;
    g.M = bp.Fp; g.N = p.Cout; g.K = BN;
    g.nparts = 3;
    g.pa[0] = 0; g.pb[0] = 0;      // f hi  d hi
    g.pa[1] = 0; g.pb[1] = 1;      // f hi  d lo
    g.pa[2] = 1; g.pb[2] = 0;      // f lo  d hi
    g.splits = bp.dw_ks;
    g.C = a.dwpart; g.ldc = p.Cout; g.zstride = (size_t)bp.Fp * p.Cout;
    g.status = ctl.status; g.timeout_ns = ctl.timeout_ns;
    if ((e = launch_bgemm(g, s)) != cudaSuccess) return e;
  }
  bwd_dw_reduce_kernel<<<cdiv((p.F + 1) * p.Cout, 256), 256, 0, s>>>(a.dwpart, io.g.w_out, io.g.b_out, p.F, bp.Fp,
                                                                      p.Cout, bp.dw_ks);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  bwd_final_kernel<<<cdiv(p.Cz * p.H + p.H, kFinalOut), 256, 0, s>>>(a);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  stage(5);
  return cudaSuccess;
}

}  // namespace fipa
