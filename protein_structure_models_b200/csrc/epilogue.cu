// epilogue.cu -- the affine output projection (features are built by the core).
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

// w_out [F, Cout] -> wT [Cout_pad, Kgp] fp16, K-major, matching the feature parts:
//   bf16 inputs: [ w | w ]            (w is exact in fp16)
//   f32  inputs: [ w hi | w lo | w hi ]
// 32 x 32 tiles transposed through shared memory (coalesced reads and writes).
template <typename T>
__global__ void __launch_bounds__(256) fipa_weight_prep_kernel(const Plan p, const T* w, __half* wT, int cout_pad) {
  __shared__ float tile[32][33];
  const int f0 = blockIdx.x * 32, n0 = blockIdx.y * 32;
  const int tx = threadIdx.x, ty = threadIdx.y;
  for (int k = ty; k < 32; k += 8) {
    const int f = f0 + k, n = n0 + tx;
    tile[k][tx] = (f < p.F && n < p.Cout) ? ld_in(w, (size_t)f * p.Cout + n) : 0.f;
  }
  __syncthreads();
  const int nseg = p.f32 ? 3 : 2;
  for (int k = ty; k < 32; k += 8) {
    const int n = n0 + k, f = f0 + tx;
    if (n >= cout_pad || f >= p.F) continue;
    const float v = tile[tx][k];
    const __half hi = __float2half_rn(v), lo = __float2half_rn(v - __half2float(hi));
    for (int seg = 0; seg < nseg; ++seg) wT[(size_t)n * p.Kgp + seg * p.F + f] = (p.f32 && seg == 1) ? lo : hi;
  }
  if (blockIdx.x == 0) {
    for (int k = ty; k < 32; k += 8) {
      const int n = n0 + k;
      if (n < cout_pad)
        for (int c = p.Kg + tx; c < p.Kgp; c += 32) wT[(size_t)n * p.Kgp + c] = __float2half_rn(0.f);
    }
  }
}

// Sum of the split-K partials, + b_out, zero for an empty neighbourhood.
template <typename T>
__global__ void fipa_proj_reduce_kernel(const Plan p, const float* part, const T* b_out, const uint8_t* rowflag,
                                        float* update) {
  const int cpad = rup(p.Cout, p.ntile_out);
  const size_t total = (size_t)p.B * p.N * p.Cout, plane = (size_t)p.B * p.N * cpad;
  for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += (size_t)gridDim.x * blockDim.x) {
    const size_t m = e / p.Cout;
    const int n = (int)(e - m * p.Cout);
    float acc = 0.f;
    for (int z = 0; z < p.gemm_ks; ++z) acc += part[z * plane + m * cpad + n];
    update[e] = rowflag[m] ? acc + ld_in(b_out, n) : 0.f;
  }
}

// ------------------------------------------------------------------ projection GEMM
struct ProjArgs {
  Plan p;
  const void* b_out;
  const uint8_t* rowflag;
  float* update;
  float* part;
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
  const int nk_all = p.Kgp / kChunk;
  const int k0 = blockIdx.z * p.gemm_nks;
  const int nk = min(nk_all, k0 + p.gemm_nks) - k0;      // K chunks of this split
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
        tma_load_2d(sa, &tmA, &full[st], (k0 + c) * kChunk, m0);
        tma_load_2d(sa + kChunkBytes, &tmB, &full[st], (k0 + c) * kChunk, n0);
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
      const int cpad = rup(p.Cout, ntile);
      float* prow = a.part + ((size_t)blockIdx.z * p.B * p.N + (size_t)m) * cpad;
      for (int c = 0; c < ntile; c += 32) {
        uint32_t o[32];
        tmem_ld32(trow + (uint32_t)c, o);
        tmem_ld_wait();
        if (live && p.gemm_ks > 1) {
#pragma unroll
          for (int e = 0; e < 32; ++e) prow[n0 + c + e] = __uint_as_float(o[e]);
        } else if (live) {
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

cudaError_t launch_weight_prep(const Plan& p, const Inputs& in, const Work& w, cudaStream_t s) {
  const int cout_pad = rup(p.Cout, p.ntile_out);
  dim3 grid((unsigned)cdiv(p.F, 32), (unsigned)cdiv(cout_pad, 32)), block(32, 8);
  if (p.f32)
    fipa_weight_prep_kernel<float><<<grid, block, 0, s>>>(p, static_cast<const float*>(in.w_out), w.wT, cout_pad);
  else
    fipa_weight_prep_kernel<__nv_bfloat16><<<grid, block, 0, s>>>(
        p, static_cast<const __nv_bfloat16*>(in.w_out), w.wT, cout_pad);
  return cudaGetLastError();
}

cudaError_t launch_out_proj(const Plan& p, const Inputs& in, const Work& w, const Outputs& out,
                            const CUtensorMap& tmA, const CUtensorMap& tmB, const DeviceCtl& ctl, cudaStream_t s) {
  ProjArgs a{p, in.b_out, w.rowflag, out.update, w.part, ctl.status, ctl.timeout_ns};
  const size_t BN = (size_t)p.B * p.N;
  dim3 grid((unsigned)((BN + kTile - 1) / kTile), (unsigned)(rup(p.Cout, p.ntile_out) / p.ntile_out),
            (unsigned)p.gemm_ks);
  cudaError_t e = allow_max_smem(reinterpret_cast<const void*>(fipa_out_proj_kernel));
  if (e != cudaSuccess) return e;
  fipa_out_proj_kernel<<<grid, 256, p.gemm_smem, s>>>(tmA, tmB, a);
  if (p.gemm_ks > 1) {
    const size_t total = BN * p.Cout;
    unsigned g = (unsigned)((total + 255) / 256);
    if (g > 148 * 16) g = 148 * 16;
    if (p.f32)
      fipa_proj_reduce_kernel<float><<<g, 256, 0, s>>>(p, w.part, static_cast<const float*>(in.b_out), w.rowflag,
                                                         out.update);
    else
      fipa_proj_reduce_kernel<__nv_bfloat16><<<g, 256, 0, s>>>(
          p, w.part, static_cast<const __nv_bfloat16*>(in.b_out), w.rowflag, out.update);
  }
  return cudaGetLastError();
}

}  // namespace fipa
