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

// w_out [F, Cout] -> wT [Cout_pad, Kgp] fp16, K-major, in the head-block order
// of the projection operand (plan.h): column k = (h * nseg + seg) * Wh8 + j
// holds row f(h, j) of w_out, f the page's head-major feature index:
//   j <  Dv           scalar   f = h*Dv + j
//   j <  Dv + 4Q      x,y,z,len  f = H*Dv + blk*H*Q + h*Q + q   (j = Dv + blk*Q + q)
//   j <  Dv + 4Q + Cz pair     f = H*Dv + 4*H*Q + h*Cz + c
// and zero for the padding j >= Wh and k >= Kg.  Segments:
//   bf16 inputs: [ w | w ]            (w is exact in fp16)
//   f32  inputs: [ w hi | w lo | w hi ]
// 32 x 32 tiles over (f, n) transposed through shared memory (coalesced reads).
__device__ __forceinline__ int feature_block_col(const Plan& p, int f, int* h) {
  const int HDv = p.H * p.Dv, HQ = p.H * p.Q;
  if (f < HDv) { *h = f / p.Dv; return f - *h * p.Dv; }
  if (f < HDv + 4 * HQ) {
    const int g = f - HDv, blk = g / HQ, rem = g - blk * HQ;
    *h = rem / p.Q;
    return p.Dv + blk * p.Q + (rem - *h * p.Q);
  }
  const int g = f - HDv - 4 * HQ;
  *h = g / p.Cz;
  return p.Dv + 4 * p.Q + (g - *h * p.Cz);
}

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
  const int f = f0 + tx;
  int h = 0;
  const int j = f < p.F ? feature_block_col(p, f, &h) : 0;
  for (int k = ty; k < 32; k += 8) {
    const int n = n0 + k;
    if (n >= cout_pad || f >= p.F) continue;
    const float v = tile[tx][k];
    const __half hi = __float2half_rn(v), lo = __float2half_rn(v - __half2float(hi));
    __half* row = wT + (size_t)n * p.Kgp + (size_t)h * p.nseg * p.Wh8 + j;
    for (int seg = 0; seg < p.nseg; ++seg) row[seg * p.Wh8] = (p.f32 && seg == 1) ? lo : hi;
  }
  if (blockIdx.x == 0) {
    // padding columns: j in [Wh, Wh8) of every head segment, and [Kg, Kgp)
    const int padw = p.Wh8 - p.Wh, nblk = p.H * p.nseg;
    for (int k = ty; k < 32; k += 8) {
      const int n = n0 + k;
      if (n >= cout_pad) continue;
      __half* row = wT + (size_t)n * p.Kgp;
      for (int e = tx; e < nblk * padw; e += 32) {
        const int bk = e / padw;
        row[(size_t)bk * p.Wh8 + p.Wh + (e - bk * padw)] = __float2half_rn(0.f);
      }
      for (int c = p.Kg + tx; c < p.Kgp; c += 32) row[c] = __float2half_rn(0.f);
    }
  }
}

// Sum of the split-K partials in split order (deterministic), + b_out, zero
// for an empty neighbourhood; 4 outputs per thread where Cout allows.
template <typename T>
__global__ void fipa_proj_reduce_kernel(const Plan p, const float* part, const T* b_out, const uint8_t* rowflag,
                                        float* update) {
  const int cpad = rup(p.Cout, p.ntile_out);
  const size_t M = (size_t)p.B * p.N, plane = M * cpad;
  const bool vec = (p.Cout & 3) == 0 && (reinterpret_cast<uintptr_t>(update) & 15) == 0;
  if (vec) {
    const int cq = p.Cout / 4;
    const size_t total = M * cq;
    for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += (size_t)gridDim.x * blockDim.x) {
      const size_t m = e / cq;
      const int n = (int)(e - m * cq) * 4;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int z = 0; z < p.gemm_ks; ++z) {
        const float4 v = *reinterpret_cast<const float4*>(part + z * plane + m * cpad + n);
        acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
      }
      const bool keep = rowflag[m] != 0;
      reinterpret_cast<float4*>(update)[e] =
          keep ? make_float4(acc.x + ld_in(b_out, n), acc.y + ld_in(b_out, n + 1), acc.z + ld_in(b_out, n + 2),
                             acc.w + ld_in(b_out, n + 3))
               : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    return;
  }
  const size_t total = M * p.Cout;
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
  }

  // ---- epilogue, all 8 warps: the accumulator goes TMEM -> registers ->
  // a staged tile in the (now idle) pipeline memory, [128][ntile + 4] fp32,
  // then out as whole rows with 16-byte stores (warps w and w+4 read the same
  // TMEM lanes and split the 32-column chunks)
  bool ok = mbar_wait(acc_full, 0, wc, 23);
  ok = __syncthreads_and(ok && *abort_flag == 0) != 0;
  tc_fence_after();
  const int sstride = ntile + 4;
  float* stile = reinterpret_cast<float*>(smem);
  if (ok) {
    const int q4 = warp & 3, half = warp >> 2;
    const int r = q4 * 32 + lane;
    const uint32_t trow = tmem + ((uint32_t)(q4 * 32) << 16);
    float* srow = stile + (size_t)r * sstride;
    for (int c = half * 32; c < ntile; c += 64) {
      uint32_t o[32];
      tmem_ld32(trow + (uint32_t)c, o);
      tmem_ld_wait();
      if (c + 32 <= ntile) {
#pragma unroll
        for (int e = 0; e < 32; e += 4)
          *reinterpret_cast<float4*>(srow + c + e) = make_float4(__uint_as_float(o[e]), __uint_as_float(o[e + 1]),
                                                                 __uint_as_float(o[e + 2]), __uint_as_float(o[e + 3]));
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e)
          if (c + e < ntile) srow[c + e] = __uint_as_float(o[e]);
      }
    }
  }
  __syncthreads();
  if (ok) {
    const int M = p.B * p.N, cpad = rup(p.Cout, ntile), nq = ntile / 4;
    const bool vec_out = (p.Cout & 3) == 0 && (reinterpret_cast<uintptr_t>(a.update) & 15) == 0;
    for (int rr = warp; rr < kTile; rr += 8) {
      const int m = m0 + rr;
      if (m >= M) break;
      const float* srow = stile + (size_t)rr * sstride;
      if (p.gemm_ks > 1) {
        float4* prow = reinterpret_cast<float4*>(a.part + ((size_t)blockIdx.z * M + m) * cpad + n0);
        for (int c4 = lane; c4 < nq; c4 += 32) prow[c4] = *reinterpret_cast<const float4*>(srow + 4 * c4);
      } else {
        const bool keep = a.rowflag[m] != 0;
        float* urow = a.update + (size_t)m * p.Cout;
        for (int c4 = lane; c4 < nq; c4 += 32) {
          const int n = n0 + 4 * c4;
          const float4 v = *reinterpret_cast<const float4*>(srow + 4 * c4);
          float w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float bo = n + e < p.Cout ? (p.f32 ? static_cast<const float*>(a.b_out)[n + e]
                                                    : __bfloat162float(static_cast<const __nv_bfloat16*>(a.b_out)[n + e]))
                                            : 0.f;
            w[e] = keep ? w[e] + bo : 0.f;
          }
          if (vec_out && n + 4 <= p.Cout) {
            *reinterpret_cast<float4*>(urow + n) = make_float4(w[0], w[1], w[2], w[3]);
          } else {
            for (int e = 0; e < 4; ++e)
              if (n + e < p.Cout) urow[n + e] = w[e];
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
