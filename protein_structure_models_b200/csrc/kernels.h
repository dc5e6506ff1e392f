// kernels.h -- argument blocks and launchers of the fused IPA forward kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <map>
#include <mutex>
#include <utility>

#include "bwd_plan.h"
#include "plan.h"

namespace fipa {

// Allow a kernel the full opt-in dynamic shared memory, once per kernel and
// device: the attribute only bounds the launch-time request, and setting it on
// every call would cost host time on every forward.
inline cudaError_t allow_max_smem(const void* kfn) {
  static std::mutex mu;
  static std::map<std::pair<const void*, int>, bool> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  auto key = std::make_pair(kfn, dev);
  if (done.count(key)) return cudaSuccess;
  int optin = 0;
  e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (e != cudaSuccess) return e;
  cudaFuncAttributes fa;
  e = cudaFuncGetAttributes(&fa, kfn);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, optin - (int)fa.sharedSizeBytes);
  if (e == cudaSuccess) done[key] = true;
  return e;
}

// Inputs exactly as the C ABI receives them (dtype fixed by Plan::f32).
struct Inputs {
  const void *q, *k, *v, *q_pts, *k_pts, *v_pts, *rot, *trans, *z1, *z2, *Wb, *raw;
  const uint8_t* mask;
  const uint8_t* pair_mask;   // may be null
  const void *w_out, *b_out;
  float eps;
};

// Workspace views (see plan.h for the layouts).
struct Work {
  __half *Q, *KH, *VH, *Z;
  float *QP, *KP;  // [B*H, N, 3P] a' and b' in fp32 (float32-input mode only)
  float4 *kvec;    // [B*H, N] {-g sum_p |b'|^2 (or -inf if masked), sum_p b'}
  float4 *qvec;    // [B*H, N] {sum_p a', -g sum_p |a'|^2}
  float4 *orig;    // [B, nG]  {32-residue group origin xyz, valid residues in group}
  int *flag;       // [B, nT]  tile has a valid residue
  float2 *stats;   // [B, H, N]  {running max M (log2 units), softmax denominator l}
  __half *feat;    // [B*N, Kgp] output-projection operand (feature hi/lo halves)
  __half *wT;      // [Cout_pad, Kgp] output-projection weights, K-major
  uint8_t *rowflag;// [B*N] row has a non-empty neighbourhood
};

struct Outputs {
  float *update, *local_points, *attention, *lse;
};

struct DeviceCtl {
  int *status;
  unsigned long long timeout_ns;
  long long *trace;   // debug event log of one core CTA, or null
  int trace_cta;
};

constexpr int kTraceCap = 4096;   // events per role of the debug trace (== FIPA_TRACE_CAP)

// Debug event log of one warp role: (event id, SM clock) pairs.
struct Tracer {
  long long* buf;
  int n;
  __device__ __forceinline__ void ev(int id) {
    if (buf != nullptr && n < kTraceCap) {
      buf[2 * n] = id;
      buf[2 * n + 1] = clock64();
      ++n;
    }
  }
};

// Launchers return the cudaError_t of the launch.
cudaError_t launch_prologue(const Plan& p, const Inputs& in, const Work& w, cudaStream_t s);
// osave: null for the forward; the backward's recompute passes its buffer of
// normalised aggregates (see CoreArgs in core.cu).
cudaError_t launch_core(const Plan& p, const Inputs& in, const Work& w, const Outputs& out,
                        const CUtensorMap& tmQ, const CUtensorMap& tmKH, const CUtensorMap& tmVH,
                        const CUtensorMap& tmZ, const DeviceCtl& ctl, cudaStream_t s, float* osave = nullptr);
cudaError_t launch_out_proj(const Plan& p, const Inputs& in, const Work& w, const Outputs& out,
                            const CUtensorMap& tmA, const CUtensorMap& tmB, const DeviceCtl& ctl,
                            cudaStream_t s);
cudaError_t launch_attention_dump(const Plan& p, const Inputs& in, const Work& w, const Outputs& out,
                                  cudaStream_t s);

// Gradient outputs of the backward pass (float32, layouts of the inputs).
struct BwdGrads {
  float *q, *k, *v, *q_pts, *k_pts, *v_pts, *rot, *trans, *z1, *z2, *Wb, *raw, *w_out, *b_out;
};
struct BwdIO {
  const float* d_update;   // [B,N,Cout] cotangent of update
  const float* d_local;    // [B,N,H,Q,3] cotangent of local_points, or null (zero)
  BwdGrads g;
  uint8_t* ws;             // workspace base (backward regions at the BwdPlan offsets)
};
// The backward kernels after the recompute (lift, and the core with the
// aggregates saved at the BwdPlan's osave offset).
// `mark(ctx, k)`, if given, is called before stage k = 1 (dfeat GEMM and prep),
// 2 (q side), 3 (k side), 4 (chain and weight gradients) and after the last (5).
typedef void (*StageMark)(void* ctx, int k);
// TMA maps of the backward's own workspace regions (encoded on the host).
struct BwdMaps {
  const CUtensorMap* dO;       // dO rows, 128-row boxes
  const CUtensorMap* Q32;      // Qhat, 32-row boxes (slices of the pair columns)
  const CUtensorMap* dO32;     // dO, 32-row boxes
  const CUtensorMap* duA[2];   // d_update hi / lo as the K-major A of dfeat (64 x 128 boxes)
  const CUtensorMap* duB[2];   // d_update hi / lo as the MN-major B of dw_out (64 x 64 boxes)
  const CUtensorMap* w[2];     // w_out hi / lo as the K-major B of dfeat (64 x 256 boxes)
  const CUtensorMap* f[2];     // feature rows hi / lo as the MN-major A of dw_out (64 x 64 boxes)
};

// The backward's dense float32 products on the tensor cores (bgemm.cu):
// C[M, N] (+ split z at C + z zstride) = sum over parts p of A_{pa[p]} B_{pb[p]}^T,
// each float32 operand as bfloat16 hi (map 0) and lo (map 1) parts.  a_mn / b_mn:
// 0 = K-major operand map (box 64 x 128 rows for A, 64 x 256 rows for B),
// 1 = MN-major (rows = K, box 64 x 64).  Splits divide K in 64-wide chunks.
struct BGemm {
  const CUtensorMap* A[2];
  const CUtensorMap* B[2];
  int a_mn, b_mn;
  int M, N, K;
  int nparts;
  int pa[3], pb[3];
  int splits;
  float* C;
  int ldc;
  size_t zstride;
  int* status;
  unsigned long long timeout_ns;
};
cudaError_t launch_bgemm(const BGemm& g, cudaStream_t s);
int bgemm_tiles(int M, int N);
// x [rows, cols] (float32, or bfloat16 when x_f32 = 0) -> bfloat16 hi, lo [rows, ldo]
cudaError_t launch_bsplit(const void* x, int x_f32, __nv_bfloat16* hi, __nv_bfloat16* lo, int rows, int cols, int ldo,
                          cudaStream_t s);

cudaError_t launch_backward(const Plan& p, const BwdPlan& bp, const Inputs& in, const Work& w, const BwdIO& io,
                            const CUtensorMap& tmQ, const CUtensorMap& tmKH, const CUtensorMap& tmVH,
                            const CUtensorMap& tmZ, const BwdMaps& bm, const DeviceCtl& ctl, cudaStream_t s,
                            StageMark mark = nullptr, void* mark_ctx = nullptr);

// The IPA layer around the core (layer.cu), float32.
cudaError_t launch_layer_proj(const float* s, const float* W_in, const float* b_in, int M, int Cs, int Din,
                              float* const dst[8], const int start[9], cudaStream_t st);
cudaError_t launch_layer_frame(const float* s, const float* upd, const float* W_bb, const float* b_bb, const float* rot,
                               const float* trans, const uint8_t* mask, int M, int Cs, float* out_s, float* out_rot,
                               float* out_trans, cudaStream_t st);

// Per-head distance weight 1/2 softplus(raw) sqrt(2/(27P)), softplus without overflow.
__device__ __forceinline__ float point_weight(float raw, int P) {
  const float sp = raw > 0.f ? raw + log1pf(expf(-raw)) : log1pf(expf(raw));
  return 0.5f * sp * sqrtf(2.0f / (27.0f * (float)P));
}

}  // namespace fipa
