// epilogue.cu -- the affine output projection (features are built by the core).
//
// Page "Invariant point attention (IPA)", Required behavior:
//   local_points_ihp = R_i^T (sum_j a_hij T_j(v_jhp) - t_i), zero for an empty
//   neighbourhood; lengths sqrt(sum_xyz local^2 + eps) (zero when empty);
//   features = [scalar (H,Dv) | x (H,Q) | y | z | lengths (H,Q) | pair (H,Cz)],
//   each flattened head-major; update = features @ w_out + b_out, zero when empty.
// The pair aggregate is rebuilt from the factors: sum_j a_ij z_ij[c] =
// sum_r z1[i,r,c] U[r,c] with U = sum_j a_ij z2[j,r,c] from the core.
#include <cooperative_groups.h>
#include <mutex>

#include "kernels.h"
#include "sm100.cuh"

namespace fipa {
namespace {

namespace cg = cooperative_groups;

// ------------------------------------------------------------------ projection GEMM
struct ProjArgs {
  Plan p;
  const void* b_out;
  const uint8_t* rowflag;
  float* update;
  int* status;
  unsigned long long timeout_ns;
  long long* trace;   // debug timeline of one CTA (last slots of the MMA role's log), or null
  int trace_cta;
  int tps;            // 0: tiles over the flattened B*N rows; else tiles per sample of the row range
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
  // output rows of this tile: [m0, min(m0 + 128, mlim))
  int m0 = blockIdx.x * kTile, mlim = p.B * p.N;
  if (a.tps > 0) {
    const int bs = blockIdx.x / a.tps, t = blockIdx.x - bs * a.tps;
    m0 = bs * p.N + p.row0 + t * kTile;
    mlim = bs * p.N + p.row1;
  }
  const int n0 = blockIdx.y * ntile;
  const bool timeline = a.trace != nullptr && threadIdx.x == 0 &&
                        (int)(blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z)) == a.trace_cta;
  Tracer ttr{timeline ? a.trace + (size_t)1 * 2 * kTraceCap : nullptr, kTraceCap - 8};
  ttr.ev(50);
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
  ttr.ev(51);

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
  ttr.ev(52);
  bool ok = mbar_wait(acc_full, 0, wc, 23);
  ttr.ev(53);
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
  // split-K across the cluster (grid z = cluster z = gemm_ks): every CTA has
  // staged its partial tile; CTA z then sums rows [z*R, (z+1)*R) of all the
  // cluster's tiles, in split order (deterministic), through distributed
  // shared memory, and writes them.  The second cluster barrier keeps every
  // tile alive until its readers are done.
  const int ks = p.gemm_ks;
  // this lane's output columns: 4-column groups c4 = lane and lane + 32 (ntile
  // <= 256); their bias is read before the barrier, off the reduce's path
  const int nq = ntile / 4;
  float bias[2][4];
#pragma unroll
  for (int u = 0; u < 2; ++u) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int n = n0 + 4 * (lane + 32 * u) + e;
      bias[u][e] = (lane + 32 * u < nq && n < p.Cout)
                       ? (p.f32 ? static_cast<const float*>(a.b_out)[n]
                                : __bfloat162float(static_cast<const __nv_bfloat16*>(a.b_out)[n]))
                       : 0.f;
    }
  }
  cg::cluster_group cluster = cg::this_cluster();
  if (ks > 1) cluster.sync();
  else __syncthreads();
  ttr.ev(54);
  if (ok) {
    const bool vec_out = (p.Cout & 3) == 0 && (reinterpret_cast<uintptr_t>(a.update) & 15) == 0;
    const int rows = (kTile + ks - 1) / ks, r0 = (int)blockIdx.z * rows, r1 = min(kTile, r0 + rows);
    for (int rr = r0 + warp; rr < r1; rr += 8) {
      const int m = m0 + rr;
      if (m >= mlim) break;
      const bool keep = a.rowflag[m] != 0;
      float* urow = a.update + (size_t)m * p.Cout;
      // every split's partial of both column groups in flight together, then
      // added in split order (deterministic)
      float4 t[2][8];
#pragma unroll
      for (int z = 0; z < 8; ++z) {
        if (z < ks) {
          const float* tz = (ks > 1 ? cluster.map_shared_rank(stile, z) : stile) + (size_t)rr * sstride;
#pragma unroll
          for (int u = 0; u < 2; ++u)
            if (lane + 32 * u < nq) t[u][z] = *reinterpret_cast<const float4*>(tz + 4 * (lane + 32 * u));
        }
      }
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int c4 = lane + 32 * u;
        if (c4 >= nq) continue;
        const int n = n0 + 4 * c4;
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int z = 0; z < 8; ++z) {
          if (z < ks) { v.x += t[u][z].x; v.y += t[u][z].y; v.z += t[u][z].z; v.w += t[u][z].w; }
        }
        float w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) w[e] = keep ? w[e] + bias[u][e] : 0.f;
        if (vec_out && n + 4 <= p.Cout) {
          *reinterpret_cast<float4*>(urow + n) = make_float4(w[0], w[1], w[2], w[3]);
        } else {
          for (int e = 0; e < 4; ++e)
            if (n + e < p.Cout) urow[n + e] = w[e];
        }
      }
    }
  }
  ttr.ev(55);
  if (ks > 1) cluster.sync();
  ttr.ev(56);
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, ncols);
  }
}

// Persistent form for many output tiles (no split-K, Cout <= one N tile):
// one CTA per SM loops over tiles t = blockIdx.x, blockIdx.x + gridDim.x, ...
// TMEM holds two accumulators, so warp 1 runs tile j+1's MMAs while warps
// 4-7 read tile j's accumulator back, add b_out (staged in shared memory
// once), zero empty rows and store whole rows as float4 from registers.
__global__ void __launch_bounds__(256, 1)
fipa_out_proj_persistent_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                                const ProjArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const Plan& p = a.p;
  const int nst = p.gemm_nst, ntile = p.ntile_out;
  const int stage = kChunkBytes + ntile * 128;
  uint8_t* tail = smem + (size_t)nst * stage;
  uint64_t* full = reinterpret_cast<uint64_t*>(tail);
  uint64_t* empty = full + 8;
  uint64_t* acc_full = full + 16;     // [2]
  uint64_t* acc_empty = full + 18;    // [2]
  uint64_t* drain = full + 20;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tail + 256);
  int* abort_flag = reinterpret_cast<int*>(tail + 260);
  float* sbias = reinterpret_cast<float*>(tail + 512);   // [ntile]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int M = p.B * p.N, tiles = (M + kTile - 1) / kTile, nk = p.Kgp / kChunk;
  const uint32_t ncols = ntile <= 32 ? 32 : ntile <= 64 ? 64 : ntile <= 128 ? 128 : 256;

  if (threadIdx.x == 0) {
    for (int st = 0; st < nst; ++st) { mbar_init(&full[st], 1); mbar_init(&empty[st], 1); }
    for (int b = 0; b < 2; ++b) { mbar_init(&acc_full[b], 1); mbar_init(&acc_empty[b], 128); }
    mbar_init(drain, 1);
    fence_mbar_init();
    *abort_flag = 0;
  }
  for (int n = threadIdx.x; n < ntile; n += blockDim.x)
    sbias[n] = n < p.Cout ? (p.f32 ? static_cast<const float*>(a.b_out)[n]
                                   : __bfloat162float(static_cast<const __nv_bfloat16*>(a.b_out)[n]))
                          : 0.f;
  if (warp == 1) { tmem_alloc(tmem_slot, 2 * ncols); tmem_relinquish(); }
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
      bool ok = true;
      for (int t = blockIdx.x; ok && t < tiles; t += gridDim.x) {
        for (int c = 0; c < nk; ++c) {
          if (!mbar_wait(&empty[st], ph ^ 1u, wc, 41)) { ok = false; break; }
          uint8_t* sa = smem + (size_t)st * stage;
          mbar_arrive_expect_tx(&full[st], (uint32_t)stage);
          tma_load_2d(sa, &tmA, &full[st], c * kChunk, t * kTile);
          tma_load_2d(sa + kChunkBytes, &tmB, &full[st], c * kChunk, 0);
          ++issued;
          if (++st == nst) { st = 0; ph ^= 1u; }
        }
      }
      if (!ok) {
        // wait (bounded) for the loads already in flight before the CTA exits
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
      bool ok = true;
      for (int t = blockIdx.x, j = 0; ok && t < tiles; t += gridDim.x, ++j) {
        const int buf = j & 1;
        if (!mbar_wait(&acc_empty[buf], ((j >> 1) & 1) ^ 1u, wc, 42)) break;
        tc_fence_after();
        const uint32_t acc = tmem + (uint32_t)(buf * ncols);
        for (int c = 0; c < nk; ++c) {
          if (!mbar_wait(&full[st], ph, wc, 43)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = smem_u32(smem + (size_t)st * stage);
          const uint32_t b0 = a0 + kChunkBytes;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ss(acc, desc_kmajor_sw128(a0 + kk * 32), desc_kmajor_sw128(b0 + kk * 32), idesc,
                   (c | kk) != 0 ? 1u : 0u);
          tc_commit(&empty[st]);
          if (++st == nst) { st = 0; ph ^= 1u; }
        }
        if (ok) tc_commit(&acc_full[buf]);
      }
      tc_commit(drain);    // fires once every MMA this thread issued is done
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(drain, 0) && global_timer_ns() - t0 < a.timeout_ns) {}
    }
  } else if (warp >= 4) {
    const int wq = warp - 4;
    const bool vec_out = (p.Cout & 3) == 0 && (reinterpret_cast<uintptr_t>(a.update) & 15) == 0;
    for (int t = blockIdx.x, j = 0; t < tiles; t += gridDim.x, ++j) {
      const int buf = j & 1;
      bool ok = mbar_wait(&acc_full[buf], (j >> 1) & 1, wc, 44);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      const int m = t * kTile + wq * 32 + lane;
      const bool live = m < M;
      const bool keep = live && a.rowflag[m] != 0;
      float* urow = a.update + (size_t)(live ? m : 0) * p.Cout;
      const uint32_t trow = tmem + (uint32_t)(buf * ncols) + ((uint32_t)(wq * 32) << 16);
      for (int c = 0; c < ntile; c += 32) {
        uint32_t o[32];
        tmem_ld32(trow + (uint32_t)c, o);
        tmem_ld_wait();
        if (!live) continue;
        float w[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) w[e] = keep ? __uint_as_float(o[e]) + sbias[c + e] : 0.f;
        if (vec_out && c + 32 <= p.Cout) {
#pragma unroll
          for (int e = 0; e < 32; e += 4)
            *reinterpret_cast<float4*>(urow + c + e) = make_float4(w[e], w[e + 1], w[e + 2], w[e + 3]);
        } else {
          for (int e = 0; e < 32; ++e)
            if (c + e < p.Cout) urow[c + e] = w[e];
        }
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[buf]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 2 * ncols);
  }
}

}  // namespace

// Largest split-K factor <= p.gemm_ks whose clusters (one per output tile, of
// ks CTAs) are all resident at once, so no tile waits for a second wave; the
// resident-cluster counts come from the occupancy API, once per device.
static int resident_split(const Plan& p, int tiles) {
  static std::mutex mu;
  static int cached[64][9] = {};          // [device][ks] max active clusters (0 = unknown)
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 1;
  const int nk = p.Kgp / kChunk;
  for (int ks = p.gemm_ks; ks > 1; --ks) {
    int n;
    {
      std::lock_guard<std::mutex> lock(mu);
      n = cached[dev][ks];
    }
    if (n == 0) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(1, 1, ks);
      cfg.blockDim = dim3(256);
      cfg.dynamicSmemBytes = p.gemm_smem;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 1;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = (unsigned)ks;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      if (cudaOccupancyMaxActiveClusters(&n, fipa_out_proj_kernel, &cfg) != cudaSuccess || n <= 0) {
        cudaGetLastError();
        n = -1;
      }
      std::lock_guard<std::mutex> lock(mu);
      cached[dev][ks] = n;
    }
    if (n > 0 && tiles <= n && cdiv(nk, ks) >= 4) return ks;
  }
  return 1;
}

cudaError_t launch_out_proj(const Plan& p, const Inputs& in, const Work& w, const Outputs& out,
                            const CUtensorMap& tmA, const CUtensorMap& tmB, const DeviceCtl& ctl, cudaStream_t s) {
  const bool full = p.row0 == 0 && p.row1 == p.N;
  const int tps = full ? 0 : cdiv(p.row1 - p.row0, kTile);
  ProjArgs a{p, in.b_out, w.rowflag, out.update, ctl.status, ctl.timeout_ns, ctl.trace, ctl.trace_cta, tps};
  const size_t BN = (size_t)p.B * p.N;
  const unsigned mt = full ? (unsigned)((BN + kTile - 1) / kTile) : (unsigned)(p.B * tps);
  const unsigned nt = (unsigned)(rup(p.Cout, p.ntile_out) / p.ntile_out);
  cudaError_t e = allow_max_smem(reinterpret_cast<const void*>(fipa_out_proj_kernel));
  if (e != cudaSuccess) return e;
  const int nk = p.Kgp / kChunk;
  if (full && p.gemm_ks == 1 && nt == 1) {
    static int sm_count[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && sm_count[dev] == 0) cudaDeviceGetAttribute(&sm_count[dev], cudaDevAttrMultiProcessorCount, dev);
    const int sms = (dev >= 0 && dev < 64 && sm_count[dev] > 0) ? sm_count[dev] : 148;
    if ((int)mt > sms) {
      const size_t smem = p.gemm_smem + 1024;           // + the staged bias
      e = cudaFuncSetAttribute(reinterpret_cast<const void*>(fipa_out_proj_persistent_kernel),
                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      fipa_out_proj_persistent_kernel<<<(unsigned)sms, 256, smem, s>>>(tmA, tmB, a);
      return cudaGetLastError();
    }
  }
  // the split-K factor of the full forward, also for a row range, so that a
  // range's rows add their K-splits exactly as the full forward does
  const int mt_full = (int)((BN + kTile - 1) / kTile);
  const int ks = p.gemm_ks > 1 ? resident_split(p, mt_full * (int)nt) : 1;
  a.p.gemm_nks = cdiv(nk, ks);
  a.p.gemm_ks = cdiv(nk, a.p.gemm_nks);
  // the split-K CTAs of one output tile form a cluster along z
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(mt, nt, (unsigned)a.p.gemm_ks);
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = p.gemm_smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = (unsigned)a.p.gemm_ks;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, fipa_out_proj_kernel, tmA, tmB, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace fipa
