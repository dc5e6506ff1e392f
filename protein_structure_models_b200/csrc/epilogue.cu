// epilogue.cu -- features and the affine output projection.
//
// Page "Invariant point attention (IPA)", Required behavior:
//   local_points_ihp = R_i^T (sum_j a_hij T_j(v_jhp) - t_i), zero for an empty
//   neighbourhood; lengths sqrt(sum_xyz local^2 + eps) (zero when empty);
//   features = [scalar (H,Dv) | x (H,Q) | y | z | lengths (H,Q) | pair (H,Cz)],
//   each flattened head-major; update = features @ w_out + b_out, zero when empty.
// The pair aggregate is rebuilt from the factors: sum_j a_ij z_ij[c] =
// sum_r z1[i,r,c] U[r,c] with U = sum_j a_ij z2[j,r,c] from the core.
#include "kernels.h"
#include "sm100.cuh"

namespace fipa {
namespace {

constexpr int kFeatWarps = 8;

struct FeatArgs {
  Plan p;
  const void* rot;
  const void* trans;
  const void* z1;
  const float* O;
  const float4* W;
  __half* feat;
  uint8_t* rowflag;
  float* local_points;
  float eps;
};

// store feature value f at feature index `col` as its 16-bit parts
__device__ __forceinline__ void put_feature(__half* row, int F, int f32, int col, float f) {
  const __half hi = __float2half_rn(f);
  const __half lo = __float2half_rn(f - __half2float(hi));
  row[col] = hi;
  if (f32) { row[F + col] = hi; row[2 * F + col] = lo; }
  else     { row[F + col] = lo; }
}

template <typename T>
__global__ void __launch_bounds__(kFeatWarps * 32) fipa_features_kernel(const FeatArgs a) {
  const Plan& p = a.p;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const size_t bi = (size_t)blockIdx.x * kFeatWarps + warp;     // residue index b*N + i
  if (bi >= (size_t)p.B * p.N) return;
  const T* rot = static_cast<const T*>(a.rot);
  const T* tr = static_cast<const T*>(a.trans);
  const T* z1 = static_cast<const T*>(a.z1);
  const int H = p.H, Dv = p.Dv, Q = p.Q, Cz = p.Cz, F = p.F, RCz = p.R * Cz;
  __half* frow = a.feat + bi * p.Kgp;
  float* lrow = a.local_points + bi * (size_t)H * Q * 3;

  const bool empty = !(a.W[bi * H].w > 0.f);     // same neighbourhood for every head
  if (lane == 0) a.rowflag[bi] = empty ? 0 : 1;
  if (empty) {
    for (int c = lane; c < p.Kgp; c += 32) frow[c] = __float2half_rn(0.f);
    for (int e = lane; e < H * Q * 3; e += 32) lrow[e] = 0.f;
    return;
  }
  for (int c = p.Kg + lane; c < p.Kgp; c += 32) frow[c] = __float2half_rn(0.f);
  float R[9], t[3];
#pragma unroll
  for (int e = 0; e < 9; ++e) R[e] = ld_in(rot, bi * 9 + e);
#pragma unroll
  for (int e = 0; e < 3; ++e) t[e] = ld_in(tr, bi * 3 + e);
  const int gofs = p.nsv * p.Dv8;
  for (int h = 0; h < H; ++h) {
    const float* orow = a.O + (bi * H + h) * p.Ocols;
    const float4 Wv = a.W[bi * H + h];
    // scalar block
    for (int d = lane; d < Dv; d += 32) {
      float s = orow[d];
      if (p.f32) s += orow[p.Dv8 + d];
      put_feature(frow, F, p.f32, h * Dv + d, s);
    }
    // points: aggregate in global frame, back into the query frame
    for (int qq = lane; qq < Q; qq += 32) {
      float G[3];
#pragma unroll
      for (int x = 0; x < 3; ++x) G[x] = orow[gofs + 3 * qq + x] + orow[gofs + p.Q38 + 3 * qq + x];
      G[0] += Wv.x - t[0];
      G[1] += Wv.y - t[1];
      G[2] += Wv.z - t[2];
      float L[3];
#pragma unroll
      for (int x = 0; x < 3; ++x) L[x] = R[0 * 3 + x] * G[0] + R[1 * 3 + x] * G[1] + R[2 * 3 + x] * G[2];
      const float len = sqrtf(L[0] * L[0] + L[1] * L[1] + L[2] * L[2] + a.eps);
      const int base = H * Dv + h * Q + qq;
      put_feature(frow, F, p.f32, base, L[0]);
      put_feature(frow, F, p.f32, base + H * Q, L[1]);
      put_feature(frow, F, p.f32, base + 2 * H * Q, L[2]);
      put_feature(frow, F, p.f32, base + 3 * H * Q, len);
      float* lp = lrow + ((size_t)h * Q + qq) * 3;
      lp[0] = L[0]; lp[1] = L[1]; lp[2] = L[2];
    }
    // pair block through the factors
    for (int c = lane; c < Cz; c += 32) {
      float acc = 0.f;
      for (int r = 0; r < p.R; ++r) {
        float u = orow[p.VHp + r * Cz + c];
        if (p.f32) u += orow[p.VHp + p.RC8 + r * Cz + c];
        acc = fmaf(ld_in(z1, bi * RCz + r * Cz + c), u, acc);
      }
      put_feature(frow, F, p.f32, H * Dv + 4 * H * Q + h * Cz + c, acc);
    }
  }
}

// w_out [F, Cout] -> wT [Cout_pad, Kgp] fp16, K-major, matching the feature parts:
//   bf16 inputs: [ w | w ]            (w is exact in fp16)
//   f32  inputs: [ w hi | w lo | w hi ]
template <typename T>
__global__ void fipa_weight_prep_kernel(const Plan p, const T* w, __half* wT, int cout_pad) {
  const size_t n_el = (size_t)cout_pad * p.Kgp;
  for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < n_el; e += (size_t)gridDim.x * blockDim.x) {
    const int n = (int)(e / p.Kgp), kk = (int)(e % p.Kgp);
    float v = 0.f;
    int is_lo = 0;
    if (n < p.Cout && kk < p.Kg) {
      const int seg = kk / p.F, f = kk - seg * p.F;
      v = ld_in(w, (size_t)f * p.Cout + n);
      is_lo = (p.f32 && seg == 1);
    }
    const __half hi = __float2half_rn(v);
    wT[e] = is_lo ? __float2half_rn(v - __half2float(hi)) : hi;
  }
}

// ------------------------------------------------------------------ projection GEMM
struct ProjArgs {
  Plan p;
  const void* b_out;
  const uint8_t* rowflag;
  float* update;
  int* status;
  unsigned long long timeout_ns;
};

// update[m, n] = sum_k feat[m, k] wT[n, k] + b_out[n], zero for empty rows.
// One CTA per 128-row x ntile tile: warp 0 streams K-chunks by TMA, warp 1
// issues tcgen05.mma into a TMEM accumulator, warps 4-7 read it back.
__global__ void __launch_bounds__(256, 1)
fipa_out_proj_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const ProjArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const Plan& p = a.p;
  const int nst = p.gemm_nst, ntile = p.ntile_out;
  const int bbytes = ntile * 128;
  const int stage = kChunkBytes + bbytes;
  uint8_t* tail = smem + (size_t)nst * stage;
  uint64_t* full = reinterpret_cast<uint64_t*>(tail);
  uint64_t* empty = full + 8;
  uint64_t* acc_full = full + 16;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tail + 256);
  int* abort_flag = reinterpret_cast<int*>(tail + 260);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * kTile, n0 = blockIdx.y * ntile;
  const int nk = p.Kgp / kChunk;
  const uint32_t ncols = ntile <= 32 ? 32 : ntile <= 64 ? 64 : ntile <= 128 ? 128 : 256;

  if (threadIdx.x == 0) {
    for (int s = 0; s < nst; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    mbar_init(acc_full, 1);
    fence_mbar_init();
    *abort_flag = 0;
  }
  if (warp == 1) { tmem_alloc(tmem_slot, ncols); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtx wc{abort_flag, a.status, a.timeout_ns};

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmB);
      int st = 0;
      uint32_t ph = 0, issued = 0;
      for (int c = 0; c < nk; ++c) {
        if (!mbar_wait(&empty[st], ph ^ 1u, wc, 21)) break;
        uint8_t* sa = smem + (size_t)st * stage;
        mbar_arrive_expect_tx(&full[st], (uint32_t)stage);
        tma_load_2d(sa, &tmA, &full[st], c * kChunk, m0);
        tma_load_2d(sa + kChunkBytes, &tmB, &full[st], c * kChunk, n0);
        ++issued;
        if (++st == nst) { st = 0; ph ^= 1u; }
      }
      if (*abort_flag) {
        const uint32_t last = issued < (uint32_t)nst ? issued : (uint32_t)nst;
        for (uint32_t k = 0; k < last; ++k) {
          const uint32_t n = issued - 1 - k;
          const uint64_t t0 = global_timer_ns();
          while (!mbar_try_wait(&full[n % nst], (n / nst) & 1u) && global_timer_ns() - t0 < a.timeout_ns) {}
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_f16(128, ntile, 0, 0);
      int st = 0;
      uint32_t ph = 0;
      for (int c = 0; c < nk; ++c) {
        if (!mbar_wait(&full[st], ph, wc, 22)) break;
        tc_fence_after();
        const uint32_t a0 = smem_u32(smem + (size_t)st * stage);
        const uint32_t b0 = a0 + kChunkBytes;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_ss(tmem, desc_kmajor_sw128(a0 + kk * 32), desc_kmajor_sw128(b0 + kk * 32), idesc,
                 (c | kk) != 0 ? 1u : 0u);
        tc_commit(&empty[st]);
        if (++st == nst) { st = 0; ph ^= 1u; }
      }
      tc_commit(acc_full);   // also the drain point: fires once all MMAs are done
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(acc_full, 0) && global_timer_ns() - t0 < a.timeout_ns) {}
    }
  } else if (warp >= 4) {
    const int wq = warp - 4;
    const int m = m0 + wq * 32 + lane;
    bool ok = mbar_wait(acc_full, 0, wc, 23);
    ok = __all_sync(0xffffffffu, ok) && !*abort_flag;
    tc_fence_after();
    if (ok) {
      const bool live = m < p.B * p.N;
      const bool keep = live && a.rowflag[m] != 0;
      const uint32_t trow = tmem + ((uint32_t)(wq * 32) << 16);
      for (int c = 0; c < ntile; c += 32) {
        uint32_t o[32];
        tmem_ld32(trow + (uint32_t)c, o);
        tmem_ld_wait();
        if (live) {
          float* urow = a.update + (size_t)m * p.Cout;
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const int n = n0 + c + e;
            if (n < p.Cout) {
              const float bo = p.f32 ? static_cast<const float*>(a.b_out)[n]
                                     : __bfloat162float(static_cast<const __nv_bfloat16*>(a.b_out)[n]);
              urow[n] = keep ? __uint_as_float(o[e]) + bo : 0.f;
            }
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, ncols);
  }
}

}  // namespace

cudaError_t launch_features(const Plan& p, const Inputs& in, const Work& w, const Outputs& out, cudaStream_t s) {
  FeatArgs a{p, in.rot, in.trans, in.z1, w.O, w.W, w.feat, w.rowflag, out.local_points, in.eps};
  const size_t BN = (size_t)p.B * p.N;
  const unsigned grid = (unsigned)((BN + kFeatWarps - 1) / kFeatWarps);
  if (p.f32) fipa_features_kernel<float><<<grid, kFeatWarps * 32, 0, s>>>(a);
  else fipa_features_kernel<__nv_bfloat16><<<grid, kFeatWarps * 32, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_weight_prep(const Plan& p, const Inputs& in, const Work& w, cudaStream_t s) {
  const int cout_pad = rup(p.Cout, p.ntile_out);
  const size_t n_el = (size_t)cout_pad * p.Kgp;
  unsigned grid = (unsigned)((n_el + 255) / 256);
  if (grid > 4096) grid = 4096;
  if (p.f32) fipa_weight_prep_kernel<float><<<grid, 256, 0, s>>>(p, static_cast<const float*>(in.w_out), w.wT, cout_pad);
  else fipa_weight_prep_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(p, static_cast<const __nv_bfloat16*>(in.w_out), w.wT, cout_pad);
  return cudaGetLastError();
}

cudaError_t launch_out_proj(const Plan& p, const Inputs& in, const Work& w, const Outputs& out,
                            const CUtensorMap& tmA, const CUtensorMap& tmB, const DeviceCtl& ctl, cudaStream_t s) {
  ProjArgs a{p, in.b_out, w.rowflag, out.update, ctl.status, ctl.timeout_ns};
  const size_t BN = (size_t)p.B * p.N;
  dim3 grid((unsigned)((BN + kTile - 1) / kTile), (unsigned)(rup(p.Cout, p.ntile_out) / p.ntile_out));
  cudaError_t e = cudaFuncSetAttribute(fipa_out_proj_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)p.gemm_smem);
  if (e != cudaSuccess) return e;
  fipa_out_proj_kernel<<<grid, 256, p.gemm_smem, s>>>(tmA, tmB, a);
  return cudaGetLastError();
}

}  // namespace fipa
