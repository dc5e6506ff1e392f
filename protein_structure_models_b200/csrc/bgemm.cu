// bgemm.cu -- the backward pass's two dense float32 products on the tensor
// cores (tcgen05, kind::f16 with bfloat16 operands, fp32 accumulation in
// tensor memory):
//   dfeat          = d_update w_out^T      M = B*N rows, N = F,    K = Cout
//   [dw_out|db_out] = featp^T d_update      M = Fp,       N = Cout, K = B*N rows
// (page "Invariant point attention (IPA)", Required behavior: update =
// features @ w_out + b_out; these are its two gradient contractions).
//
// Every float32 operand x travels as two bfloat16 numbers, hi = bf16(x) and
// lo = bf16(x - hi): |x - hi - lo| <= 2^-18 |x| with float32's exponent range.
// A product is the sum of the hi*hi, hi*lo and lo*hi parts (the lo*lo part is
// below 2^-17 relative and dropped); an exact bfloat16 operand (w_out given in
// bfloat16) has no lo part.
#include "kernels.h"
#include "sm100.cuh"

namespace fipa {
namespace {

constexpr int kGemmNT = 256;                     // N tile (accumulator columns)
constexpr int kGemmStages = 4;
constexpr int kGemmABytes = 128 * 64 * 2;         // 128 M-rows x 64 K, bf16
constexpr int kGemmBBytes = kGemmNT * 64 * 2;     // 256 N-rows x 64 K, bf16
constexpr int kGemmStage = kGemmABytes + kGemmBBytes;
constexpr int kGemmBox = 64 * 64 * 2;             // one 64 x 64 MN-major box

struct GemmArgs {
  int M, N, K;          // C[M, N] = sum over parts of A_a[M, K] B_b[N, K]^T
  int nparts;
  int pa[3], pb[3];     // part p multiplies A map pa[p] by B map pb[p] (0 = hi, 1 = lo)
  int kc_per_split;     // 64-wide K chunks per split (blockIdx.z)
  float* C;
  int ldc;
  size_t zstride;       // split z writes C + z * zstride
  int* status;
  unsigned long long timeout_ns;
};

__device__ __forceinline__ void gemm_drain(uint64_t* bar, uint32_t parity, uint64_t timeout_ns) {
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > timeout_ns) break;
  }
}

// A_MN / B_MN: 0 = K-major operand (memory rows = M or N, K contiguous; one box
// of 64 K x 128 (A) or 256 (B) rows), 1 = MN-major (memory rows = K; boxes of
// 64 M/N x 64 K, 8 KB apart).  One CTA per (M tile, N tile, K split): warp 0
// streams the parts' chunks by TMA, warp 1 issues the MMAs, warps 4-7 move the
// accumulator to C.
template <int A_MN, int B_MN>
__global__ void __launch_bounds__(256, 1)
bgemm_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmA1,
             const __grid_constant__ CUtensorMap tmB0, const __grid_constant__ CUtensorMap tmB1,
             const GemmArgs g) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* tail = smem + (size_t)kGemmStages * kGemmStage;
  uint64_t* full = reinterpret_cast<uint64_t*>(tail);
  uint64_t* empty = full + kGemmStages;
  uint64_t* acc_full = empty + kGemmStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tail + 128);
  int* abort_flag = reinterpret_cast<int*>(tail + 132);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * 128, n0 = blockIdx.y * kGemmNT;
  const int nkc = (g.K + 63) / 64;
  const int kc0 = blockIdx.z * g.kc_per_split;
  const int kc1 = min(nkc, kc0 + g.kc_per_split);
  const int nsteps = kc1 > kc0 ? (kc1 - kc0) * g.nparts : 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kGemmStages; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    mbar_init(acc_full, 1);
    fence_mbar_init();
    *abort_flag = 0;
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kGemmNT);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtx wc{abort_flag, g.status, g.timeout_ns};

  if (warp == 0) {
    if (lane == 0 && nsteps > 0) {
      tma_prefetch_desc(&tmA0);
      tma_prefetch_desc(&tmA1);
      tma_prefetch_desc(&tmB0);
      tma_prefetch_desc(&tmB1);
      int st = 0;
      uint32_t ph = 0;
      int issued = 0;
      for (int step = 0; step < nsteps; ++step) {
        const int kc = kc0 + step / g.nparts, part = step % g.nparts;
        if (!mbar_wait(&empty[st], ph ^ 1u, wc, 71)) break;
        mbar_arrive_expect_tx(&full[st], (uint32_t)kGemmStage);
        uint8_t* sa = smem + (size_t)st * kGemmStage;
        uint8_t* sb = sa + kGemmABytes;
        const CUtensorMap* ta = g.pa[part] ? &tmA1 : &tmA0;
        const CUtensorMap* tb = g.pb[part] ? &tmB1 : &tmB0;
        const int k0 = kc * 64;
        if (A_MN) {
          tma_load_2d(sa, ta, &full[st], m0, k0);
          tma_load_2d(sa + kGemmBox, ta, &full[st], m0 + 64, k0);
        } else {
          tma_load_2d(sa, ta, &full[st], k0, m0);
        }
        if (B_MN) {
#pragma unroll
          for (int q = 0; q < kGemmNT / 64; ++q) tma_load_2d(sb + q * kGemmBox, tb, &full[st], n0 + 64 * q, k0);
        } else {
          tma_load_2d(sb, tb, &full[st], k0, n0);
        }
        ++issued;
        if (++st == kGemmStages) { st = 0; ph ^= 1u; }
      }
      if (*abort_flag) {
        // let the loads in flight land before the CTA's shared memory is released
        const int last = issued < kGemmStages ? issued : kGemmStages;
        for (int k = 0; k < last; ++k) {
          const int n = issued - 1 - k;
          gemm_drain(&full[n % kGemmStages], (uint32_t)(n / kGemmStages) & 1u, g.timeout_ns);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && nsteps > 0) {
      const uint32_t idesc = idesc_bf16(128, kGemmNT, A_MN, B_MN);
      int st = 0;
      uint32_t ph = 0;
      for (int step = 0; step < nsteps; ++step) {
        if (!mbar_wait(&full[st], ph, wc, 72)) break;
        tc_fence_after();
        const uint32_t sa = smem_u32(smem + (size_t)st * kGemmStage), sb = sa + kGemmABytes;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t ad = A_MN ? desc_mnmajor_sw128(sa + kk * 2048, kGemmBox) : desc_kmajor_sw128(sa + kk * 32);
          const uint64_t bd = B_MN ? desc_mnmajor_sw128(sb + kk * 2048, kGemmBox) : desc_kmajor_sw128(sb + kk * 32);
          mma_ss(tmem, ad, bd, idesc, (step > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(&empty[st]);
        if (++st == kGemmStages) { st = 0; ph ^= 1u; }
      }
      tc_commit(acc_full);
      gemm_drain(acc_full, 0, g.timeout_ns);
    }
  } else if (warp >= 4) {
    // accumulator row r = TMEM lane r -> C row m0 + r; a split without K chunks writes zeros
    const int wq = warp - 4;
    const int r = wq * 32 + lane;
    const int m = m0 + r;
    bool ok = true;
    if (nsteps > 0) {
      ok = mbar_wait(acc_full, 0, wc, 73);
      ok = __all_sync(0xffffffffu, ok);
      tc_fence_after();
    }
    const bool aborted = __any_sync(0xffffffffu, *abort_flag != 0);
    float* crow = g.C + blockIdx.z * g.zstride + (size_t)(m < g.M ? m : 0) * g.ldc;
    for (int c0 = 0; c0 < kGemmNT; c0 += 32) {
      if (n0 + c0 >= g.N) break;                                      // uniform over the CTA
      uint32_t v[32];
      if (nsteps > 0 && ok && !aborted) {
        tmem_ld32(tmem + ((uint32_t)(wq * 32) << 16) + (uint32_t)c0, v);
        tmem_ld_wait();
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] = 0u;
      }
      if (m < g.M && !aborted) {
        const int nn = n0 + c0;
        if (nn + 32 <= g.N && (g.ldc & 3) == 0) {
          float4* c4 = reinterpret_cast<float4*>(crow + nn);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            c4[e] = make_float4(__uint_as_float(v[4 * e]), __uint_as_float(v[4 * e + 1]),
                                __uint_as_float(v[4 * e + 2]), __uint_as_float(v[4 * e + 3]));
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (nn + e < g.N) crow[nn + e] = __uint_as_float(v[e]);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kGemmNT);
  }
}

// x (float32 or bfloat16, [rows, cols]) -> hi, lo (bfloat16, [rows, ldo]),
// zero in the padding columns [cols, ldo).
__global__ void bsplit_kernel(const void* __restrict__ x, int x_f32, __nv_bfloat16* __restrict__ hi,
                              __nv_bfloat16* __restrict__ lo, int rows, int cols, int ldo) {
  const size_t n = (size_t)rows * ldo;
  for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (size_t)gridDim.x * blockDim.x) {
    const int r = (int)(e / ldo), c = (int)(e - (size_t)r * ldo);
    float v = 0.f;
    if (c < cols) {
      const size_t i = (size_t)r * cols + c;
      v = x_f32 ? static_cast<const float*>(x)[i] : __bfloat162float(static_cast<const __nv_bfloat16*>(x)[i]);
    }
    const __nv_bfloat16 h = __float2bfloat16_rn(v);
    hi[e] = h;
    lo[e] = __float2bfloat16_rn(v - __bfloat162float(h));
  }
}

template <int A_MN, int B_MN>
cudaError_t launch_one(const BGemm& b, const GemmArgs& g, dim3 grid, cudaStream_t s) {
  const size_t smem = 1024 + (size_t)kGemmStages * kGemmStage + 256;
  cudaError_t e = cudaFuncSetAttribute(bgemm_kernel<A_MN, B_MN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  bgemm_kernel<A_MN, B_MN><<<grid, 256, smem, s>>>(*b.A[0], *b.A[1], *b.B[0], *b.B[1], g);
  return cudaGetLastError();
}

}  // namespace

size_t bgemm_split_grid(size_t n) {
  const size_t blocks = (n + 255) / 256;
  return blocks < 148 * 16 ? blocks : 148 * 16;
}

cudaError_t launch_bsplit(const void* x, int x_f32, __nv_bfloat16* hi, __nv_bfloat16* lo, int rows, int cols, int ldo,
                          cudaStream_t s) {
  const size_t n = (size_t)rows * ldo;
  if (n == 0) return cudaSuccess;
  bsplit_kernel<<<(unsigned)bgemm_split_grid(n), 256, 0, s>>>(x, x_f32, hi, lo, rows, cols, ldo);
  return cudaGetLastError();
}

int bgemm_tiles(int M, int N) { return ((M + 127) / 128) * ((N + kGemmNT - 1) / kGemmNT); }

cudaError_t launch_bgemm(const BGemm& b, cudaStream_t s) {
  GemmArgs g;
  g.M = b.M; g.N = b.N; g.K = b.K;
  g.nparts = b.nparts;
  for (int p = 0; p < 3; ++p) { g.pa[p] = b.pa[p]; g.pb[p] = b.pb[p]; }
  const int nkc = (b.K + 63) / 64;
  const int ks = b.splits < 1 ? 1 : (b.splits > nkc ? nkc : b.splits);
  g.kc_per_split = (nkc + ks - 1) / ks;
  g.C = b.C; g.ldc = b.ldc; g.zstride = b.zstride;
  g.status = b.status; g.timeout_ns = b.timeout_ns;
  const dim3 grid((unsigned)((b.M + 127) / 128), (unsigned)((b.N + kGemmNT - 1) / kGemmNT), (unsigned)b.splits);
  if (b.a_mn == 0 && b.b_mn == 0) return launch_one<0, 0>(b, g, grid, s);
  if (b.a_mn == 1 && b.b_mn == 1) return launch_one<1, 1>(b, g, grid, s);
  return cudaErrorInvalidValue;
}

}  // namespace fipa
