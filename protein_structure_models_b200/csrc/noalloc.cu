// noalloc.cu -- fipa_forward_noalloc: the fused IPA forward for callers that
// cannot allocate device memory on their call path.
//
// Who needs it: plugins whose host framework owns every device allocation
// through its own pool and hands the plugin none, and latency-bound callers
// that may not call cudaMalloc at run time (it can synchronise the device and
// can fail under memory pressure in the middle of a step).  Such callers
// cannot call cudaMalloc for a workspace, nor fipa_create (which allocates the
// handle's status word).  This entry point needs neither: its scratch is one
// fixed file-scope device array of FIPA_NOALLOC_SCRATCH_BYTES, held by every
// GPU that loads this library until the process exits, and its device status
// word is a file-scope variable too.
//
// The kernels and their launch order are those of fipa_forward; only where the
// workspace comes from differs.
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "fipa.h"
#include "kernels.h"

#define FIPA_API extern "C" __attribute__((visibility("default")))

namespace {

// The scratch array and the device status word of this entry point.  In host
// code these names are host-side stand-ins, not device addresses: their device
// addresses come from cudaGetSymbolAddress (see device_state below).
static __device__ __align__(256) uint8_t g_noalloc_scratch[FIPA_NOALLOC_SCRATCH_BYTES];
static __device__ __align__(16) int g_noalloc_status[4];

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

constexpr int kMaxDevices = 64;
struct DeviceState {
  bool ready = false;
  uint8_t* scratch = nullptr;   // device address of g_noalloc_scratch on this device
  int* status = nullptr;        // device address of g_noalloc_status on this device
  unsigned long long timeout_ns = 2000000000ull;   // budget of every bounded device wait
};
std::mutex g_mu;
DeviceState g_state[kMaxDevices];
EncodeTiledFn g_encode = nullptr;

// Once per device, with that device current: resolve the device addresses of
// the file-scope arrays (and, once per process, the tensor-map encoder).
fipa_status device_state(int dev, DeviceState** out) {
  if (dev < 0 || dev >= kMaxDevices) return FIPA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState& st = g_state[dev];
  if (!st.ready) {
    // the kernels are built for sm_100a only
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return FIPA_ERR_CUDA;
    if (major != 10 || minor != 0) return FIPA_ERR_UNSUPPORTED;
    // same wait budget as fipa_create: FIPA_WAIT_TIMEOUT_MS, read once per device
    if (const char* env = std::getenv("FIPA_WAIT_TIMEOUT_MS")) {
      const long ms = std::strtol(env, nullptr, 10);
      if (ms > 0) st.timeout_ns = (unsigned long long)ms * 1000000ull;
    }
    if (g_encode == nullptr) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
          q != cudaDriverEntryPointSuccess || fn == nullptr)
        return FIPA_ERR_CUDA;
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    }
    void* s = nullptr;
    void* w = nullptr;
    if (cudaGetSymbolAddress(&s, g_noalloc_scratch) != cudaSuccess) return FIPA_ERR_CUDA;
    if (cudaGetSymbolAddress(&w, g_noalloc_status) != cudaSuccess) return FIPA_ERR_CUDA;
    st.scratch = static_cast<uint8_t*>(s);
    st.status = static_cast<int*>(w);
    st.ready = true;
  }
  *out = &st;
  return FIPA_OK;
}

fipa_status encode(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint64_t outer,
                   uint32_t box_rows, cuuint32_t rank) {
  cuuint64_t dims[3] = {cols, rows, outer};
  cuuint64_t strides[2] = {cols * 2, cols * rows * 2};
  cuuint32_t box[3] = {64, box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, rank, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FIPA_OK : FIPA_ERR_CUDA;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// True when `p` is device (or managed) memory that device `dev` owns.  The
// scratch address and the launches belong to the current device, so inputs on
// another device are rejected before anything runs.
bool on_device(const void* p, int dev) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();   // an unknown pointer leaves a (non-sticky) error behind: clear it
    return false;
  }
  return (a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged) && a.device == dev;
}

}  // namespace

FIPA_API fipa_status fipa_forward_noalloc(fipa_dtype dtype, const void* q, const void* k, const void* v,
                                          const void* q_pts, const void* k_pts, const void* v_pts, const void* rot,
                                          const void* trans, const void* z1, const void* z2, const void* Wb,
                                          const void* point_w_raw, const uint8_t* mask, const uint8_t* pair_mask,
                                          const void* w_out, const void* b_out, double eps, const fipa_dims* dims,
                                          float* out_update, float* out_local_points, float* out_lse,
                                          void* stream) {
  if (dtype != FIPA_F32 && dtype != FIPA_BF16) return FIPA_ERR_INVALID_ARG;
  if (dims == nullptr) return FIPA_ERR_INVALID_ARG;
  fipa::Plan p;
  const char* why = "";
  const int rc = fipa::make_plan(p, dims->B, dims->N, dims->H, dims->D, dims->Dv, dims->P, dims->Q, dims->Cz,
                                 dims->R, dims->Cout, dtype == FIPA_F32 ? 1 : 0, &why);
  if (rc == 1) return FIPA_ERR_INVALID_ARG;
  if (rc == 2) return FIPA_ERR_UNSUPPORTED;
  if (p.total > (size_t)FIPA_NOALLOC_SCRATCH_BYTES) return FIPA_ERR_WORKSPACE;   // problem too large
  const size_t es = dtype == FIPA_F32 ? 4 : 2;
  const void* req[] = {q, k, v, q_pts, k_pts, v_pts, rot, trans, z1, z2, Wb, point_w_raw, w_out, b_out};
  for (const void* ptr : req)
    if (ptr == nullptr || !aligned(ptr, es)) return FIPA_ERR_INVALID_ARG;
  if (mask == nullptr || out_update == nullptr || out_local_points == nullptr) return FIPA_ERR_INVALID_ARG;
  if (!aligned(out_update, 4) || !aligned(out_local_points, 4) || !aligned(out_lse, 4)) return FIPA_ERR_INVALID_ARG;
  if (!(eps > 0.0) || !std::isfinite(eps)) return FIPA_ERR_INVALID_ARG;

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FIPA_ERR_CUDA;
  DeviceState* ds = nullptr;
  fipa_status st = device_state(dev, &ds);
  if (st != FIPA_OK) return st;
  if (!on_device(q, dev) || !on_device(out_update, dev)) return FIPA_ERR_INVALID_ARG;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = ds->scratch;
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

  fipa::Inputs in{q, k, v, q_pts, k_pts, v_pts, rot, trans, z1, z2, Wb, point_w_raw, mask, pair_mask,
                  w_out, b_out, (float)eps};
  fipa::Outputs out{out_update, out_local_points, nullptr, out_lse};
  fipa::DeviceCtl ctl{ds->status, ds->timeout_ns, nullptr, -1};
  const uint64_t BH = (uint64_t)p.B * p.H, N = (uint64_t)p.N, B = (uint64_t)p.B;

  CUtensorMap tmQ, tmKH, tmVH, tmZ, tmA, tmB;
  if (encode(&tmQ, w.Q, p.Kq, N, BH, 128, 3) != FIPA_OK || encode(&tmKH, w.KH, p.KHp, N, BH, 128, 3) != FIPA_OK ||
      encode(&tmVH, w.VH, p.VHp, N, BH, 128, 3) != FIPA_OK || encode(&tmZ, w.Z, p.Zp, N, B, 128, 3) != FIPA_OK ||
      encode(&tmA, w.feat, p.Kgp, B * N, 1, 128, 2) != FIPA_OK ||
      encode(&tmB, w.wT, p.Kgp, (uint64_t)fipa::rup(p.Cout, p.ntile_out), 1, p.ntile_out, 2) != FIPA_OK)
    return FIPA_ERR_CUDA;

  // the status word must start at zero; nothing in the scratch needs clearing
  // (every kernel writes all of what a later kernel reads)
  if (cudaMemsetAsync(ds->status, 0, sizeof(int), s) != cudaSuccess) return FIPA_ERR_CUDA;
  if (fipa::launch_prologue(p, in, w, s) != cudaSuccess) return FIPA_ERR_CUDA;
  if (fipa::launch_core(p, in, w, out, tmQ, tmKH, tmVH, tmZ, ctl, s) != cudaSuccess) return FIPA_ERR_CUDA;
  if (fipa::launch_out_proj(p, in, w, out, tmA, tmB, ctl, s) != cudaSuccess) return FIPA_ERR_CUDA;
  return FIPA_OK;
}
