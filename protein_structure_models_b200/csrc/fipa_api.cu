// fipa_api.cu -- the C ABI of include/fipa.h: validation, planning, TMA
// descriptors and kernel launches.  No allocation per call, no host sync in
// fipa_forward, status codes instead of exceptions.
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <string>

#include "fipa.h"
#include "kernels.h"
#include "sm100.cuh"

#define FIPA_API extern "C" __attribute__((visibility("default")))

using fipa::Plan;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// stage-timing intervals: prologue, core, output projection, attention output
constexpr int kStages = FIPA_STAGES;
// backward: recompute, prep, q side, k side, chain and weight gradients
constexpr int kBwdStages = FIPA_BWD_STAGES;

struct fipa_handle {
  int device = 0;
  fipa_dtype dtype = FIPA_BF16;
  bool has_max = false;
  fipa_dims max_dims{};
  int* d_status = nullptr;
  unsigned long long timeout_ns = 2000000000ull;
  EncodeTiledFn encode = nullptr;
  std::string last_error;
  bool timing = false;
  bool timed_call = false;
  cudaEvent_t ev[kStages + 1] = {};
  cudaEvent_t bev[kBwdStages + 1] = {};   // backward stage events (with stage timing on)
  bool bwd_timed_call = false;
  long long* d_trace = nullptr;
  int trace_cta = -1;
  int pair_split = 1;
  int value_buffer = 1;
  int ring_cap = 8;
  // TMA descriptors of the last call: they depend only on the workspace
  // address and the dims, so a loop over the same buffers encodes them once
  struct MapCache {
    bool valid = false;
    const void* ws = nullptr;
    fipa_dims dims{};
    int sig[5] = {0, 0, 0, 0, 0};   // layout widths the maps were encoded for
    CUtensorMap Q, KH, VH, Z, A, B;
  } maps;
  // the backward's maps, cached the same way: dO with 128-row boxes, Qhat and
  // dO with 32-row boxes (the k side's slices of the pair columns), and the
  // bfloat16 hi / lo operands of its two dense products
  struct BwdMapCache {
    bool valid = false;
    const void* ws = nullptr;
    fipa_dims dims{};
    CUtensorMap dO, Q32, dO32, duA[2], duB[2], w[2], f[2];
  } bmaps;
};

namespace {

struct DeviceGuard {
  int prev = -1, want;
  explicit DeviceGuard(int d) : want(d) {
    if (cudaGetDevice(&prev) != cudaSuccess) prev = -1;
    if (prev != want) cudaSetDevice(want);
  }
  ~DeviceGuard() {
    if (prev >= 0 && prev != want) cudaSetDevice(prev);
  }
};

fipa_status fail(fipa_handle* h, fipa_status s, const std::string& msg) {
  if (h != nullptr) h->last_error = msg;
  return s;
}

fipa_status cuda_fail(fipa_handle* h, const char* what, cudaError_t e) {
  return fail(h, FIPA_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// 16-bit row-major tensor [outer, rows, cols] as a TMA map with a 64 x `box_rows`
// box and 128-byte swizzle (cols is a multiple of 64, so rows are 128-B aligned).
fipa_status encode_rows(fipa_handle* h, CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows,
                        uint64_t outer, uint32_t box_rows, cuuint32_t rank, const char* what) {
  cuuint64_t dims[3] = {cols, rows, outer};
  cuuint64_t strides[2] = {cols * 2, cols * rows * 2};
  cuuint32_t box[3] = {64, box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = h->encode(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, rank, const_cast<void*>(base), dims, strides, box,
                         estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(h, FIPA_ERR_CUDA, std::string("cuTensorMapEncodeTiled failed for ") + what + " (" +
                                      std::to_string((int)r) + ")");
  return FIPA_OK;
}

// Work views of a workspace (plan.h layout).
fipa::Work work_views(const Plan& p, void* workspace) {
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  fipa::Work w;
  w.Q = reinterpret_cast<__half*>(ws + p.off_Q);
  w.KH = reinterpret_cast<__half*>(ws + p.off_KH);
  w.VH = reinterpret_cast<__half*>(ws + p.off_VH);
  w.Z = reinterpret_cast<__half*>(ws + p.off_Z);
  w.QP = reinterpret_cast<float*>(ws + p.off_QP);
  w.KP = reinterpret_cast<float*>(ws + p.off_KP);
  w.kvec = reinterpret_cast<float4*>(ws + p.off_kvec);
  w.qvec = reinterpret_cast<float4*>(ws + p.off_qvec);
  w.orig = reinterpret_cast<float4*>(ws + p.off_orig);
  w.flag = reinterpret_cast<int*>(ws + p.off_flag);
  w.stats = reinterpret_cast<float2*>(ws + p.off_stats);
  w.feat = reinterpret_cast<__half*>(ws + p.off_feat);
  w.wT = reinterpret_cast<__half*>(ws + p.off_wT);
  w.rowflag = ws + p.off_rowflag;
  return w;
}

// TMA descriptors of the lifted rows, the features and the prepared weights:
// they depend only on the workspace address and the dims, so a loop over the
// same buffers encodes them once.
fipa_status ensure_maps(fipa_handle* h, const Plan& p, const fipa::Work& w, const void* workspace,
                        const fipa_dims* dims) {
  const uint64_t BH = (uint64_t)p.B * p.H, N = (uint64_t)p.N, B = (uint64_t)p.B;
  fipa_handle::MapCache& mc = h->maps;
  const int sig[5] = {p.Kq, p.KHp, p.VHp, p.Zp, p.Kgp};
  if (!mc.valid || mc.ws != workspace || std::memcmp(&mc.dims, dims, sizeof(fipa_dims)) != 0 ||
      std::memcmp(mc.sig, sig, sizeof(sig)) != 0) {
    mc.valid = false;
    fipa_status st;
    if ((st = encode_rows(h, &mc.Q, w.Q, p.Kq, N, BH, 128, 3, "Qhat")) != FIPA_OK) return st;
    if ((st = encode_rows(h, &mc.KH, w.KH, p.KHp, N, BH, 128, 3, "Khat")) != FIPA_OK) return st;
    if ((st = encode_rows(h, &mc.VH, w.VH, p.VHp, N, BH, 128, 3, "Vhat")) != FIPA_OK) return st;
    if ((st = encode_rows(h, &mc.Z, w.Z, p.Zp, N, B, 128, 3, "Z")) != FIPA_OK) return st;
    if ((st = encode_rows(h, &mc.A, w.feat, p.Kgp, B * N, 1, 128, 2, "features")) != FIPA_OK) return st;
    if ((st = encode_rows(h, &mc.B, w.wT, p.Kgp, (uint64_t)fipa::rup(p.Cout, p.ntile_out), 1, p.ntile_out, 2,
                          "w_out")) != FIPA_OK)
      return st;
    mc.ws = workspace;
    mc.dims = *dims;
    std::memcpy(mc.sig, sig, sizeof(sig));
    mc.valid = true;
  }
  return FIPA_OK;
}

int plan_for(fipa_handle* h, const fipa_dims* d, Plan& p) {
  const char* why = "";
  int rc = fipa::make_plan(p, d->B, d->N, d->H, d->D, d->Dv, d->P, d->Q, d->Cz, d->R, d->Cout,
                           h->dtype == FIPA_F32 ? 1 : 0, &why, h->pair_split, h->value_buffer, h->ring_cap);
  if (rc != 0) h->last_error = why;
  return rc;
}

// The forward plan the backward recomputes with: the bfloat16 lifted layout
// (fp16 products), reading the handle's input dtype.  float32 inputs are thus
// differentiated at the backward's fp16-product precision.
int bwd_plan_for(fipa_handle* h, const fipa_dims* d, Plan& p) {
  const char* why = "";
  int rc = fipa::make_plan(p, d->B, d->N, d->H, d->D, d->Dv, d->P, d->Q, d->Cz, d->R, d->Cout, 0, &why,
                           h->pair_split, h->value_buffer, h->ring_cap);
  if (rc != 0) {
    h->last_error = why;
    return rc;
  }
  p.in_f32 = h->dtype == FIPA_F32 ? 1 : 0;
  return 0;
}

}  // namespace

FIPA_API const char* fipa_status_string(fipa_status s) {
  switch (s) {
    case FIPA_OK: return "ok";
    case FIPA_ERR_INVALID_ARG: return "invalid argument";
    case FIPA_ERR_UNSUPPORTED: return "unsupported configuration";
    case FIPA_ERR_WORKSPACE: return "workspace missing or too small";
    case FIPA_ERR_CUDA: return "CUDA error";
    case FIPA_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
    case FIPA_ERR_INTERNAL: return "internal error";
  }
  return "unknown status";
}

FIPA_API const char* fipa_last_error(const fipa_handle* h) {
  return h == nullptr ? "" : h->last_error.c_str();
}

FIPA_API fipa_status fipa_create(fipa_handle** out, const fipa_dims* max_dims, fipa_dtype dtype, int device) {
  if (out == nullptr) return FIPA_ERR_INVALID_ARG;
  *out = nullptr;
  if (dtype != FIPA_F32 && dtype != FIPA_BF16) return FIPA_ERR_INVALID_ARG;
  if (device < 0) return FIPA_ERR_INVALID_ARG;
  if (max_dims != nullptr) {
    const int* f = &max_dims->B;
    for (int k = 0; k < 10; ++k)
      if (f[k] <= 0) return FIPA_ERR_INVALID_ARG;
  }
  int count = 0;
  if (cudaGetDeviceCount(&count) != cudaSuccess || device >= count) return FIPA_ERR_CUDA;
  int major = 0, minor = 0;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, device);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, device);
  if (major != 10 || minor != 0) return FIPA_ERR_UNSUPPORTED;   // built for sm_100a only
  fipa_handle* h = new (std::nothrow) fipa_handle();
  if (h == nullptr) return FIPA_ERR_INTERNAL;
  h->device = device;
  h->dtype = dtype;
  if (max_dims != nullptr) { h->has_max = true; h->max_dims = *max_dims; }
  if (const char* env = std::getenv("FIPA_WAIT_TIMEOUT_MS")) {
    const long ms = std::strtol(env, nullptr, 10);
    if (ms > 0) h->timeout_ns = (unsigned long long)ms * 1000000ull;
  }
  DeviceGuard g(device);
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess || fn == nullptr) {
    delete h;
    return FIPA_ERR_CUDA;
  }
  h->encode = reinterpret_cast<EncodeTiledFn>(fn);
  if (const char* env = std::getenv("FIPA_PAIR_SPLIT")) h->pair_split = std::strtol(env, nullptr, 10) != 0;
  if (const char* env = std::getenv("FIPA_VALUE_BUFFER")) {
    const long v = std::strtol(env, nullptr, 10);
    h->value_buffer = v <= 0 ? 0 : (v >= 2 ? 2 : 1);
  }
  if (const char* env = std::getenv("FIPA_RING_STAGES")) {
    const long v = std::strtol(env, nullptr, 10);
    if (v >= 2 && v <= 8) h->ring_cap = (int)v;
  }
  if (const char* env = std::getenv("FIPA_TRACE_CTA")) {
    h->trace_cta = (int)std::strtol(env, nullptr, 10);
    const size_t bytes = (size_t)4 * FIPA_TRACE_CAP * 2 * sizeof(long long);
    if (cudaMalloc(&h->d_trace, bytes) != cudaSuccess) { delete h; return FIPA_ERR_CUDA; }
  }
  if (cudaMalloc(&h->d_status, 256) != cudaSuccess || cudaMemset(h->d_status, 0, 256) != cudaSuccess ||
      cudaDeviceSynchronize() != cudaSuccess) {
    if (h->d_status) cudaFree(h->d_status);
    delete h;
    return FIPA_ERR_CUDA;
  }
  *out = h;
  return FIPA_OK;
}

FIPA_API fipa_status fipa_enable_stage_timing(fipa_handle* h, int enable) {
  if (h == nullptr) return FIPA_ERR_INVALID_ARG;
  DeviceGuard g(h->device);
  if (enable && !h->timing) {
    for (auto& e : h->ev) {
      cudaError_t err = cudaEventCreate(&e);
      if (err != cudaSuccess) return cuda_fail(h, "event create", err);
    }
    for (auto& e : h->bev) {
      cudaError_t err = cudaEventCreate(&e);
      if (err != cudaSuccess) return cuda_fail(h, "event create", err);
    }
    h->timing = true;
  } else if (!enable && h->timing) {
    for (auto& e : h->ev) { cudaEventDestroy(e); e = nullptr; }
    for (auto& e : h->bev) { cudaEventDestroy(e); e = nullptr; }
    h->timing = false;
  }
  h->timed_call = false;
  h->bwd_timed_call = false;
  return FIPA_OK;
}

FIPA_API fipa_status fipa_stage_times(fipa_handle* h, float* ms, int n) {
  if (h == nullptr || ms == nullptr || n < 0) return FIPA_ERR_INVALID_ARG;
  if (!h->timing || !h->timed_call) return fail(h, FIPA_ERR_INVALID_ARG, "no timed fipa_forward call");
  DeviceGuard g(h->device);
  cudaError_t e = cudaEventSynchronize(h->ev[kStages]);
  if (e != cudaSuccess) return cuda_fail(h, "event sync", e);
  for (int k = 0; k < kStages && k < n; ++k) {
    float t = 0.f;
    e = cudaEventElapsedTime(&t, h->ev[k], h->ev[k + 1]);
    if (e != cudaSuccess) return cuda_fail(h, "event time", e);
    ms[k] = t;
  }
  return FIPA_OK;
}

FIPA_API fipa_status fipa_destroy(fipa_handle* h) {
  if (h == nullptr) return FIPA_OK;
  {
    DeviceGuard g(h->device);
    if (h->d_status) cudaFree(h->d_status);
    if (h->d_trace) cudaFree(h->d_trace);
    if (h->timing) {
      for (auto& e : h->ev) cudaEventDestroy(e);
      for (auto& e : h->bev) cudaEventDestroy(e);
    }
  }
  delete h;
  return FIPA_OK;
}

FIPA_API fipa_status fipa_workspace_size(const fipa_handle* hc, const fipa_dims* dims, size_t* bytes) {
  fipa_handle* h = const_cast<fipa_handle*>(hc);
  if (h == nullptr || dims == nullptr || bytes == nullptr) return fail(h, FIPA_ERR_INVALID_ARG, "null argument");
  Plan p;
  const int rc = plan_for(h, dims, p);
  if (rc == 1) return FIPA_ERR_INVALID_ARG;
  if (rc == 2) return FIPA_ERR_UNSUPPORTED;
  *bytes = p.total;
  return FIPA_OK;
}

FIPA_API fipa_status fipa_trace_copy(fipa_handle* h, int64_t* host, size_t n_values, void* stream) {
  if (h == nullptr || host == nullptr) return FIPA_ERR_INVALID_ARG;
  const size_t need = (size_t)4 * FIPA_TRACE_CAP * 2;
  if (h->d_trace == nullptr || n_values < need) return fail(h, FIPA_ERR_INVALID_ARG, "tracing is off or buffer too small");
  DeviceGuard g(h->device);
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(h, "stream", e);
  e = cudaMemcpy(host, h->d_trace, need * sizeof(long long), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(h, "trace copy", e);
  return FIPA_OK;
}

FIPA_API fipa_status fipa_kernel_count(const fipa_handle* hc, const fipa_dims* dims, int with_attention,
                                       int* count) {
  fipa_handle* h = const_cast<fipa_handle*>(hc);
  if (h == nullptr || dims == nullptr || count == nullptr) return fail(h, FIPA_ERR_INVALID_ARG, "null argument");
  Plan p;
  const int rc = plan_for(h, dims, p);
  if (rc == 1) return FIPA_ERR_INVALID_ARG;
  if (rc == 2) return FIPA_ERR_UNSUPPORTED;
  // prologue (weight prep + lift), core, projection (+ attention)
  *count = 3 + (with_attention ? 1 : 0);
  return FIPA_OK;
}

FIPA_API fipa_status fipa_sync_status(fipa_handle* h, void* stream) {
  if (h == nullptr) return FIPA_ERR_INVALID_ARG;
  DeviceGuard g(h->device);
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(h, "stream", e);
  int code = 0;
  e = cudaMemcpy(&code, h->d_status, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(h, "status read", e);
  if (code != 0) {
    cudaMemset(h->d_status, 0, sizeof(int));
    char buf[96];
    std::snprintf(buf, sizeof(buf), "device wait timed out (code %d, site %d)", code & 0xff, code >> 8);
    return fail(h, FIPA_ERR_DEVICE_TIMEOUT, buf);
  }
  return FIPA_OK;
}

namespace {
// One CTA whose thread 0 waits, with the library's bounded wait, on an
// mbarrier that nothing ever completes: the wait runs out, raises the CTA's
// abort flag, writes the timeout code into the status word and returns.
__global__ void fipa_selftest_wait_kernel(int* status, unsigned long long timeout_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    fipa::mbar_init(&bar, 1);
    fipa::fence_mbar_init();
    abort_flag = 0;
    const fipa::WaitCtx wc{&abort_flag, status, timeout_ns};
    fipa::mbar_wait(&bar, 0, wc, 63);
  }
}
}  // namespace

FIPA_API fipa_status fipa_selftest_timeout(fipa_handle* h, unsigned timeout_ms, void* stream) {
  if (h == nullptr || timeout_ms == 0 || timeout_ms > 10000) return FIPA_ERR_INVALID_ARG;
  DeviceGuard g(h->device);
  fipa_selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      h->d_status, (unsigned long long)timeout_ms * 1000000ull);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(h, "self-test launch", e);
  return FIPA_OK;
}

// The forward over query rows [row0, row1) of every sample (row1 < 0: N).
static fipa_status forward_impl(fipa_handle* h, const void* q, const void* k, const void* v, const void* q_pts,
                                const void* k_pts, const void* v_pts, const void* rot, const void* trans,
                                const void* z1, const void* z2, const void* Wb, const void* point_w_raw,
                                const uint8_t* mask, const uint8_t* pair_mask, const void* w_out,
                                const void* b_out, double eps, const fipa_dims* dims, int row0, int row1,
                                float* out_update, float* out_local_points, float* out_attention, float* out_lse,
                                void* workspace, size_t workspace_bytes, void* stream, float* osave = nullptr) {
  if (h == nullptr) return FIPA_ERR_INVALID_ARG;
  h->last_error.clear();
  if (dims == nullptr) return fail(h, FIPA_ERR_INVALID_ARG, "dims is NULL");
  Plan p;
  const int rc = plan_for(h, dims, p);
  if (rc == 1) return FIPA_ERR_INVALID_ARG;
  if (rc == 2) return FIPA_ERR_UNSUPPORTED;
  if (row1 < 0) row1 = p.N;
  if (row0 < 0 || row0 >= row1 || row1 > p.N || row0 % fipa::kTile != 0 || (row1 % fipa::kTile != 0 && row1 != p.N))
    return fail(h, FIPA_ERR_INVALID_ARG,
                "row range must satisfy 0 <= row_begin < row_end <= N, row_begin a multiple of 128, "
                "row_end a multiple of 128 or N");
  p.row0 = row0;
  p.row1 = row1;
  if (h->has_max) {
    const int* a = &dims->B;
    const int* m = &h->max_dims.B;
    for (int i = 0; i < 10; ++i)
      if (a[i] > m[i]) return fail(h, FIPA_ERR_INVALID_ARG, "dims exceed the handle's max_dims");
  }
  const size_t es = h->dtype == FIPA_F32 ? 4 : 2;
  const void* req[] = {q, k, v, q_pts, k_pts, v_pts, rot, trans, z1, z2, Wb, point_w_raw, w_out, b_out};
  const char* names[] = {"q", "k", "v", "q_pts", "k_pts", "v_pts", "rot", "trans", "z1", "z2", "Wb",
                         "point_w_raw", "w_out", "b_out"};
  for (int i = 0; i < 14; ++i) {
    if (req[i] == nullptr) return fail(h, FIPA_ERR_INVALID_ARG, std::string(names[i]) + " is NULL");
    if (!aligned(req[i], es)) return fail(h, FIPA_ERR_INVALID_ARG, std::string(names[i]) + " is misaligned");
  }
  if (mask == nullptr) return fail(h, FIPA_ERR_INVALID_ARG, "mask is NULL");
  if (out_update == nullptr || out_local_points == nullptr)
    return fail(h, FIPA_ERR_INVALID_ARG, "out_update / out_local_points is NULL");
  if (!aligned(out_update, 4) || !aligned(out_local_points, 4) || !aligned(out_attention, 4) || !aligned(out_lse, 4))
    return fail(h, FIPA_ERR_INVALID_ARG, "output pointer misaligned");
  if (!(eps > 0.0) || !std::isfinite(eps)) return fail(h, FIPA_ERR_INVALID_ARG, "eps must be finite and > 0");
  if (workspace == nullptr || workspace_bytes < p.total)
    return fail(h, FIPA_ERR_WORKSPACE, "workspace needs " + std::to_string(p.total) + " bytes");
  if (!aligned(workspace, 256)) return fail(h, FIPA_ERR_INVALID_ARG, "workspace must be 256-byte aligned");

  DeviceGuard g(h->device);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const fipa::Work w = work_views(p, workspace);

  fipa::Inputs in{q, k, v, q_pts, k_pts, v_pts, rot, trans, z1, z2, Wb, point_w_raw, mask, pair_mask,
                  w_out, b_out, (float)eps};
  fipa::Outputs out{out_update, out_local_points, out_attention, out_lse};
  fipa::DeviceCtl ctl{h->d_status, h->timeout_ns, h->d_trace, h->trace_cta};
  if (h->d_trace != nullptr) cudaMemsetAsync(h->d_trace, 0xff, (size_t)4 * FIPA_TRACE_CAP * 2 * sizeof(long long), s);
  fipa_status mst = ensure_maps(h, p, w, workspace, dims);
  if (mst != FIPA_OK) return mst;
  fipa_handle::MapCache& mc = h->maps;
  const CUtensorMap &tmQ = mc.Q, &tmKH = mc.KH, &tmVH = mc.VH, &tmZ = mc.Z, &tmA = mc.A, &tmB = mc.B;

  cudaError_t e;
  const bool rec = h->timing;
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (rec) cudaStreamIsCapturing(s, &cap);
  // inside a stream capture the events become event-record nodes of the graph,
  // so each replay re-records them and fipa_stage_times reads the replay
  const unsigned rec_flags = cap == cudaStreamCaptureStatusActive ? cudaEventRecordExternal : cudaEventRecordDefault;
  auto mark = [&](int k) {
    if (rec) cudaEventRecordWithFlags(h->ev[k], s, rec_flags);
  };
  mark(0);
  if ((e = fipa::launch_prologue(p, in, w, s)) != cudaSuccess) return cuda_fail(h, "prologue launch", e);
  mark(1);
  if ((e = fipa::launch_core(p, in, w, out, tmQ, tmKH, tmVH, tmZ, ctl, s, osave)) != cudaSuccess)
    return cuda_fail(h, "core launch", e);
  mark(2);
  if ((e = fipa::launch_out_proj(p, in, w, out, tmA, tmB, ctl, s)) != cudaSuccess)
    return cuda_fail(h, "output projection launch", e);
  mark(3);
  if (out_attention != nullptr) {
    if ((e = fipa::launch_attention_dump(p, in, w, out, s)) != cudaSuccess)
      return cuda_fail(h, "attention launch", e);
  }
  mark(4);
  h->timed_call = rec;
  return FIPA_OK;
}

FIPA_API fipa_status fipa_forward(fipa_handle* h, const void* q, const void* k, const void* v, const void* q_pts,
                                  const void* k_pts, const void* v_pts, const void* rot, const void* trans,
                                  const void* z1, const void* z2, const void* Wb, const void* point_w_raw,
                                  const uint8_t* mask, const uint8_t* pair_mask, const void* w_out,
                                  const void* b_out, double eps, const fipa_dims* dims, float* out_update,
                                  float* out_local_points, float* out_attention, float* out_lse, void* workspace,
                                  size_t workspace_bytes, void* stream) {
  return forward_impl(h, q, k, v, q_pts, k_pts, v_pts, rot, trans, z1, z2, Wb, point_w_raw, mask, pair_mask, w_out,
                      b_out, eps, dims, 0, -1, out_update, out_local_points, out_attention, out_lse, workspace,
                      workspace_bytes, stream);
}

FIPA_API fipa_status fipa_forward_rows(fipa_handle* h, const void* q, const void* k, const void* v,
                                       const void* q_pts, const void* k_pts, const void* v_pts, const void* rot,
                                       const void* trans, const void* z1, const void* z2, const void* Wb,
                                       const void* point_w_raw, const uint8_t* mask, const uint8_t* pair_mask,
                                       const void* w_out, const void* b_out, double eps, const fipa_dims* dims,
                                       int row_begin, int row_end, float* out_update, float* out_local_points,
                                       float* out_attention, float* out_lse, void* workspace,
                                       size_t workspace_bytes, void* stream) {
  return forward_impl(h, q, k, v, q_pts, k_pts, v_pts, rot, trans, z1, z2, Wb, point_w_raw, mask, pair_mask, w_out,
                      b_out, eps, dims, row_begin, row_end, out_update, out_local_points, out_attention, out_lse,
                      workspace, workspace_bytes, stream);
}

// ---------------------------------------------------------------- backward
FIPA_API fipa_status fipa_backward_workspace_size(const fipa_handle* hc, const fipa_dims* dims, size_t* bytes) {
  fipa_handle* h = const_cast<fipa_handle*>(hc);
  if (h == nullptr || dims == nullptr || bytes == nullptr) return fail(h, FIPA_ERR_INVALID_ARG, "null argument");
  Plan p;
  const int rc = bwd_plan_for(h, dims, p);
  if (rc == 1) return FIPA_ERR_INVALID_ARG;
  if (rc == 2) return FIPA_ERR_UNSUPPORTED;
  fipa::BwdPlan bp;
  const char* why = "";
  if (fipa::make_bwd_plan(bp, p, &why) != 0) return fail(h, FIPA_ERR_UNSUPPORTED, why);
  *bytes = bp.total;
  return FIPA_OK;
}

static fipa_status backward_impl(fipa_handle* h, const void* q, const void* k, const void* v, const void* q_pts,
                                 const void* k_pts, const void* v_pts, const void* rot, const void* trans,
                                 const void* z1, const void* z2, const void* Wb, const void* point_w_raw,
                                 const uint8_t* mask, const uint8_t* pair_mask, const void* w_out,
                                 const void* b_out, double eps, const fipa_dims* dims, const float* d_update,
                                 const float* d_local_points, const fipa_grads* grads, void* workspace,
                                 size_t workspace_bytes, void* stream, bool recompute) {
  if (h == nullptr) return FIPA_ERR_INVALID_ARG;
  h->last_error.clear();
  if (dims == nullptr) return fail(h, FIPA_ERR_INVALID_ARG, "dims is NULL");
  if (h->dtype != FIPA_BF16 && !recompute)
    return fail(h, FIPA_ERR_UNSUPPORTED, "the backward from saved state supports bfloat16 inputs only");
  Plan p;
  const int rc = bwd_plan_for(h, dims, p);
  if (rc == 1) return FIPA_ERR_INVALID_ARG;
  if (rc == 2) return FIPA_ERR_UNSUPPORTED;
  if (h->has_max) {
    const int* a = &dims->B;
    const int* m = &h->max_dims.B;
    for (int i = 0; i < 10; ++i)
      if (a[i] > m[i]) return fail(h, FIPA_ERR_INVALID_ARG, "dims exceed the handle's max_dims");
  }
  fipa::BwdPlan bp;
  const char* why = "";
  if (fipa::make_bwd_plan(bp, p, &why) != 0) return fail(h, FIPA_ERR_UNSUPPORTED, why);
  const void* req[] = {q, k, v, q_pts, k_pts, v_pts, rot, trans, z1, z2, Wb, point_w_raw, w_out, b_out};
  const char* names[] = {"q", "k", "v", "q_pts", "k_pts", "v_pts", "rot", "trans", "z1", "z2", "Wb",
                         "point_w_raw", "w_out", "b_out"};
  const size_t ies = h->dtype == FIPA_F32 ? 4 : 2;
  for (int i = 0; i < 14; ++i) {
    if (req[i] == nullptr) return fail(h, FIPA_ERR_INVALID_ARG, std::string(names[i]) + " is NULL");
    if (!aligned(req[i], ies)) return fail(h, FIPA_ERR_INVALID_ARG, std::string(names[i]) + " is misaligned");
  }
  if (mask == nullptr) return fail(h, FIPA_ERR_INVALID_ARG, "mask is NULL");
  if (d_update == nullptr || !aligned(d_update, 4) || !aligned(d_local_points, 4))
    return fail(h, FIPA_ERR_INVALID_ARG, "d_update is NULL or a cotangent is misaligned");
  if (grads == nullptr) return fail(h, FIPA_ERR_INVALID_ARG, "grads is NULL");
  float* const outs[] = {grads->q, grads->k, grads->v, grads->q_pts, grads->k_pts, grads->v_pts, grads->rot,
                         grads->trans, grads->z1, grads->z2, grads->Wb, grads->point_w_raw, grads->w_out,
                         grads->b_out};
  for (int i = 0; i < 14; ++i)
    if (outs[i] == nullptr || !aligned(outs[i], 4))
      return fail(h, FIPA_ERR_INVALID_ARG, std::string("gradient of ") + names[i] + " is NULL or misaligned");
  if (!(eps > 0.0) || !std::isfinite(eps)) return fail(h, FIPA_ERR_INVALID_ARG, "eps must be finite and > 0");
  if (workspace == nullptr || workspace_bytes < bp.total)
    return fail(h, FIPA_ERR_WORKSPACE, "backward workspace needs " + std::to_string(bp.total) + " bytes");
  if (!aligned(workspace, 256)) return fail(h, FIPA_ERR_INVALID_ARG, "workspace must be 256-byte aligned");

  DeviceGuard g(h->device);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const fipa::Work w = work_views(p, workspace);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* osave = reinterpret_cast<float*>(ws + bp.off_osave);
  fipa::Inputs in{q, k, v, q_pts, k_pts, v_pts, rot, trans, z1, z2, Wb, point_w_raw, mask, pair_mask,
                  w_out, b_out, (float)eps};
  fipa::Outputs out{nullptr, reinterpret_cast<float*>(ws + bp.off_lp), nullptr, nullptr};
  fipa::DeviceCtl ctl{h->d_status, h->timeout_ns, nullptr, -1};
  fipa_status mst = ensure_maps(h, p, w, workspace, dims);
  if (mst != FIPA_OK) return mst;
  fipa_handle::BwdMapCache& bm = h->bmaps;
  if (!bm.valid || bm.ws != workspace || std::memcmp(&bm.dims, dims, sizeof(fipa_dims)) != 0) {
    bm.valid = false;
    const uint64_t BH = (uint64_t)p.B * p.H;
    if ((mst = encode_rows(h, &bm.dO, ws + bp.off_dO, bp.Vw, (uint64_t)p.N, BH, 128, 3, "dO")) != FIPA_OK ||
        (mst = encode_rows(h, &bm.dO32, ws + bp.off_dO, bp.Vw, (uint64_t)p.N, BH, 32, 3, "dO slices")) != FIPA_OK ||
        (mst = encode_rows(h, &bm.Q32, w.Q, p.Kq, (uint64_t)p.N, BH, 32, 3, "Qhat slices")) != FIPA_OK)
      return mst;
    const uint64_t BN = (uint64_t)p.B * p.N;
    const size_t du_off[2] = {bp.off_duhi, bp.off_dulo}, w_off[2] = {bp.off_whi, bp.off_wlo},
                 f_off[2] = {bp.off_fhi, bp.off_flo};
    for (int k = 0; k < 2; ++k) {
      if ((mst = encode_rows(h, &bm.duA[k], ws + du_off[k], bp.Coutp, BN, 1, 128, 2, "d_update parts")) != FIPA_OK ||
          (mst = encode_rows(h, &bm.duB[k], ws + du_off[k], bp.Coutp, BN, 1, 64, 2, "d_update parts")) != FIPA_OK ||
          (mst = encode_rows(h, &bm.w[k], ws + w_off[k], bp.Coutp, (uint64_t)p.F, 1, 256, 2, "w_out parts")) !=
              FIPA_OK ||
          (mst = encode_rows(h, &bm.f[k], ws + f_off[k], bp.Fp, BN, 1, 64, 2, "feature parts")) != FIPA_OK)
        return mst;
    }
    bm.ws = workspace;
    bm.dims = *dims;
    bm.valid = true;
  }
  const fipa_handle::MapCache& mc = h->maps;
  fipa::BwdIO io{d_update, d_local_points,
                 fipa::BwdGrads{grads->q, grads->k, grads->v, grads->q_pts, grads->k_pts, grads->v_pts, grads->rot,
                                grads->trans, grads->z1, grads->z2, grads->Wb, grads->point_w_raw, grads->w_out,
                                grads->b_out},
                 ws};
  cudaError_t e;
  struct Marker {
    fipa_handle* h;
    cudaStream_t s;
    unsigned flags;
  } mk{h, s, cudaEventRecordDefault};
  const bool rec = h->timing;
  if (rec) {
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    cudaStreamIsCapturing(s, &cap);
    mk.flags = cap == cudaStreamCaptureStatusActive ? cudaEventRecordExternal : cudaEventRecordDefault;
  }
  auto mark = [](void* ctx, int k) {
    Marker* m = static_cast<Marker*>(ctx);
    cudaEventRecordWithFlags(m->h->bev[k], m->s, m->flags);
  };
  if (rec) mark(&mk, 0);
  if (recompute) {
    // recompute: the lift, and the core saving the normalised aggregates
    if ((e = fipa::launch_prologue(p, in, w, s)) != cudaSuccess) return cuda_fail(h, "prologue launch", e);
    if ((e = fipa::launch_core(p, in, w, out, mc.Q, mc.KH, mc.VH, mc.Z, ctl, s, osave)) != cudaSuccess)
      return cuda_fail(h, "core launch", e);
  }
  const fipa::BwdMaps maps{&bm.dO, &bm.Q32, &bm.dO32, {&bm.duA[0], &bm.duA[1]}, {&bm.duB[0], &bm.duB[1]},
                           {&bm.w[0], &bm.w[1]}, {&bm.f[0], &bm.f[1]}};
  if ((e = fipa::launch_backward(p, bp, in, w, io, mc.Q, mc.KH, mc.VH, mc.Z, maps, ctl, s,
                                 rec ? +mark : nullptr, &mk)) != cudaSuccess)
    return cuda_fail(h, "backward launch", e);
  h->bwd_timed_call = rec;
  return FIPA_OK;
}

FIPA_API fipa_status fipa_backward(fipa_handle* h, const void* q, const void* k, const void* v, const void* q_pts,
                                   const void* k_pts, const void* v_pts, const void* rot, const void* trans,
                                   const void* z1, const void* z2, const void* Wb, const void* point_w_raw,
                                   const uint8_t* mask, const uint8_t* pair_mask, const void* w_out,
                                   const void* b_out, double eps, const fipa_dims* dims, const float* d_update,
                                   const float* d_local_points, const fipa_grads* grads, void* workspace,
                                   size_t workspace_bytes, void* stream) {
  return backward_impl(h, q, k, v, q_pts, k_pts, v_pts, rot, trans, z1, z2, Wb, point_w_raw, mask, pair_mask,
                       w_out, b_out, eps, dims, d_update, d_local_points, grads, workspace, workspace_bytes, stream,
                       true);
}

FIPA_API fipa_status fipa_backward_saved(fipa_handle* h, const void* q, const void* k, const void* v,
                                         const void* q_pts, const void* k_pts, const void* v_pts, const void* rot,
                                         const void* trans, const void* z1, const void* z2, const void* Wb,
                                         const void* point_w_raw, const uint8_t* mask, const uint8_t* pair_mask,
                                         const void* w_out, const void* b_out, double eps, const fipa_dims* dims,
                                         const float* d_update, const float* d_local_points,
                                         const fipa_grads* grads, void* workspace, size_t workspace_bytes,
                                         void* stream) {
  return backward_impl(h, q, k, v, q_pts, k_pts, v_pts, rot, trans, z1, z2, Wb, point_w_raw, mask, pair_mask,
                       w_out, b_out, eps, dims, d_update, d_local_points, grads, workspace, workspace_bytes, stream,
                       false);
}

FIPA_API fipa_status fipa_forward_train(fipa_handle* h, const void* q, const void* k, const void* v,
                                        const void* q_pts, const void* k_pts, const void* v_pts, const void* rot,
                                        const void* trans, const void* z1, const void* z2, const void* Wb,
                                        const void* point_w_raw, const uint8_t* mask, const uint8_t* pair_mask,
                                        const void* w_out, const void* b_out, double eps, const fipa_dims* dims,
                                        float* out_update, float* out_local_points, float* out_lse, void* workspace,
                                        size_t workspace_bytes, void* stream) {
  if (h == nullptr) return FIPA_ERR_INVALID_ARG;
  if (dims == nullptr) return fail(h, FIPA_ERR_INVALID_ARG, "dims is NULL");
  if (h->dtype != FIPA_BF16) return fail(h, FIPA_ERR_UNSUPPORTED, "the backward pass supports bfloat16 inputs only");
  Plan p;
  const int rc = plan_for(h, dims, p);
  if (rc == 1) return FIPA_ERR_INVALID_ARG;
  if (rc == 2) return FIPA_ERR_UNSUPPORTED;
  fipa::BwdPlan bp;
  const char* why = "";
  if (fipa::make_bwd_plan(bp, p, &why) != 0) return fail(h, FIPA_ERR_UNSUPPORTED, why);
  if (workspace == nullptr || workspace_bytes < bp.total)
    return fail(h, FIPA_ERR_WORKSPACE, "training workspace needs " + std::to_string(bp.total) + " bytes");
  float* osave = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + bp.off_osave);
  return forward_impl(h, q, k, v, q_pts, k_pts, v_pts, rot, trans, z1, z2, Wb, point_w_raw, mask, pair_mask, w_out,
                      b_out, eps, dims, 0, -1, out_update, out_local_points, nullptr, out_lse, workspace,
                      workspace_bytes, stream, osave);
}

FIPA_API fipa_status fipa_backward_stage_times(fipa_handle* h, float* ms, int n) {
  if (h == nullptr || ms == nullptr || n < 0) return FIPA_ERR_INVALID_ARG;
  if (!h->timing || !h->bwd_timed_call) return fail(h, FIPA_ERR_INVALID_ARG, "no timed fipa_backward call");
  DeviceGuard g(h->device);
  cudaError_t e = cudaEventSynchronize(h->bev[kBwdStages]);
  if (e != cudaSuccess) return cuda_fail(h, "event sync", e);
  for (int k = 0; k < kBwdStages && k < n; ++k) {
    float t = 0.f;
    e = cudaEventElapsedTime(&t, h->bev[k], h->bev[k + 1]);
    if (e != cudaSuccess) return cuda_fail(h, "event time", e);
    ms[k] = t;
  }
  return FIPA_OK;
}

// ---------------------------------------------------------------- IPA layer
namespace {
struct LayerLayout {
  int Din;
  int start[9];
  size_t off_blk[8], off_upd, total;
};

void layer_layout(const Plan& p, LayerLayout& L) {
  const int widths[8] = {p.H * p.D, p.H * p.D, p.H * p.Dv, p.H * p.P * 3, p.H * p.P * 3, p.H * p.Q * 3,
                         p.R * p.Cz, p.R * p.Cz};
  const size_t BN = (size_t)p.B * p.N;
  L.start[0] = 0;
  size_t o = fipa::rup_sz(p.total, 256);
  for (int i = 0; i < 8; ++i) {
    L.start[i + 1] = L.start[i] + widths[i];
    L.off_blk[i] = o;
    o = fipa::rup_sz(o + BN * widths[i] * 4, 256);
  }
  L.Din = L.start[8];
  L.off_upd = o;
  o = fipa::rup_sz(o + BN * p.Cout * 4, 256);
  L.total = o;
}
}  // namespace

FIPA_API fipa_status fipa_layer_workspace_size(const fipa_handle* hc, const fipa_dims* dims, size_t* bytes) {
  fipa_handle* h = const_cast<fipa_handle*>(hc);
  if (h == nullptr || dims == nullptr || bytes == nullptr) return fail(h, FIPA_ERR_INVALID_ARG, "null argument");
  Plan p;
  const int rc = plan_for(h, dims, p);
  if (rc == 1) return FIPA_ERR_INVALID_ARG;
  if (rc == 2) return FIPA_ERR_UNSUPPORTED;
  LayerLayout L;
  layer_layout(p, L);
  *bytes = L.total;
  return FIPA_OK;
}

FIPA_API fipa_status fipa_ipa_layer(fipa_handle* h, const float* s, const float* W_in, const float* b_in,
                                    const float* rot, const float* trans, const uint8_t* mask,
                                    const uint8_t* pair_mask, const float* Wb, const float* point_w_raw,
                                    const float* w_out, const float* b_out, const float* W_bb, const float* b_bb,
                                    double eps, const fipa_dims* dims, float* out_s, float* out_rot,
                                    float* out_trans, float* out_local_points, void* workspace,
                                    size_t workspace_bytes, void* stream) {
  if (h == nullptr) return FIPA_ERR_INVALID_ARG;
  h->last_error.clear();
  if (dims == nullptr) return fail(h, FIPA_ERR_INVALID_ARG, "dims is NULL");
  if (h->dtype != FIPA_F32) return fail(h, FIPA_ERR_UNSUPPORTED, "the IPA layer runs with a float32 handle");
  Plan p;
  const int rc = plan_for(h, dims, p);
  if (rc == 1) return FIPA_ERR_INVALID_ARG;
  if (rc == 2) return FIPA_ERR_UNSUPPORTED;
  const void* req[] = {s, W_in, b_in, rot, trans, mask, Wb, point_w_raw, w_out, b_out, W_bb, b_bb,
                       out_s, out_rot, out_trans, out_local_points};
  for (const void* ptr : req)
    if (ptr == nullptr) return fail(h, FIPA_ERR_INVALID_ARG, "a required pointer is NULL");
  const void* al[] = {s, W_in, b_in, rot, trans, Wb, point_w_raw, w_out, b_out, W_bb, b_bb, out_s, out_rot,
                      out_trans, out_local_points};
  for (const void* ptr : al)
    if (!aligned(ptr, 4)) return fail(h, FIPA_ERR_INVALID_ARG, "a float pointer is misaligned");
  LayerLayout L;
  layer_layout(p, L);
  if (workspace == nullptr || workspace_bytes < L.total)
    return fail(h, FIPA_ERR_WORKSPACE, "layer workspace needs " + std::to_string(L.total) + " bytes");
  if (!aligned(workspace, 256)) return fail(h, FIPA_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  DeviceGuard g(h->device);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* blk[8];
  for (int i = 0; i < 8; ++i) blk[i] = reinterpret_cast<float*>(ws + L.off_blk[i]);
  float* upd = reinterpret_cast<float*>(ws + L.off_upd);
  const int M = p.B * p.N;
  cudaError_t e;
  if ((e = fipa::launch_layer_proj(s, W_in, b_in, M, p.Cout, L.Din, blk, L.start, st)) != cudaSuccess)
    return cuda_fail(h, "layer projection launch", e);
  fipa_status fs = forward_impl(h, blk[0], blk[1], blk[2], blk[3], blk[4], blk[5], rot, trans, blk[6], blk[7], Wb,
                                point_w_raw, mask, pair_mask, w_out, b_out, eps, dims, 0, -1, upd, out_local_points,
                                nullptr, nullptr, workspace, p.total, stream);
  if (fs != FIPA_OK) return fs;
  if ((e = fipa::launch_layer_frame(s, upd, W_bb, b_bb, rot, trans, mask, M, p.Cout, out_s, out_rot, out_trans,
                                    st)) != cudaSuccess)
    return cuda_fail(h, "layer frame-update launch", e);
  return FIPA_OK;
}
