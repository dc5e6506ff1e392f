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
  float* O;
  float4* W;
  float2* stats;
  float* lse;
  int* status;
  unsigned long long timeout_ns;
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
constexpr int kOkBuf = 256;        // 2 x 4 key-group origins (float4)
constexpr int kMisc = 384;         // tmem slot, abort flag, tile count
constexpr int kKtBuf = 1024;       // 2 x 4 query groups x 128 keys per-key terms (floats)
constexpr int kTiles = 5120;       // uint16 key-tile list (<= 1024 entries)
constexpr int kKpBuf = 7168;       // fp32 key points of two key tiles (float32-input mode)

__device__ __forceinline__ float load_raw(const CoreArgs& a, int h) {
  return a.p.f32 ? static_cast<const float*>(a.raw)[h]
                 : __bfloat162float(static_cast<const __nv_bfloat16*>(a.raw)[h]);
}

// Bounded wait that ignores the abort flag (used only to drain in-flight work).
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity, uint64_t timeout_ns) {
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > timeout_ns) break;
  }
}

template <bool SPLIT>
__global__ void __launch_bounds__(256, 1)
fipa_core_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmKH,
                 const __grid_constant__ CUtensorMap tmVH, const __grid_constant__ CUtensorMap tmZ,
                 const CoreArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const Plan& p = a.p;
  uint8_t* sQ = smem;
  uint8_t* sRing = sQ + p.nQc * kChunkBytes;
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
  float* ktbuf = reinterpret_cast<float*>(tail + kKtBuf);
  float4* okbuf = reinterpret_cast<float4*>(tail + kOkBuf);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tail + kMisc);
  int* abort_flag = reinterpret_cast<int*>(tail + kMisc + 4);
  int* ntiles = reinterpret_cast<int*>(tail + kMisc + 8);
  uint16_t* tiles = reinterpret_cast<uint16_t*>(tail + kTiles);
  float* kpbuf = reinterpret_cast<float*>(tail + kKpBuf);          // [2][128][3P] (SPLIT only)

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
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

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && nkt > 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmKH);
      tma_prefetch_desc(&tmVH);
      tma_prefetch_desc(&tmZ);
      mbar_arrive_expect_tx(q_full, (uint32_t)(p.nQc * kChunkBytes));
      for (int c = 0; c < p.nQc; ++c) tma_load_3d(sQ + c * kChunkBytes, &tmQ, q_full, c * kChunk, qt * kTile, bh);
      int st = 0;
      uint32_t ph = 0;
      bool ok = true;
      uint32_t issued = 0;
      auto push = [&](const CUtensorMap* tm, int c0, int c1, int c2) {
        if (!ok) return;
        if (!mbar_wait(&empty[st], ph ^ 1u, wc, 1)) { ok = false; return; }
        mbar_arrive_expect_tx(&full[st], kChunkBytes);
        tma_load_3d(sRing + st * kChunkBytes, tm, &full[st], c0, c1, c2);
        ++issued;
        if (++st == p.nst) { st = 0; ph ^= 1u; }
      };
      auto push_qk = [&](int kt) {
        for (int c = 0; c < p.nZ; ++c) push(&tmZ, c * kChunk, kt * kTile, b);
        for (int c = 0; c < p.nKH; ++c) push(&tmKH, c * kChunk, kt * kTile, bh);
      };
      auto push_pv = [&](int kt) {
        for (int c = 0; c < p.nVH; ++c) push(&tmVH, c * kChunk, kt * kTile, bh);
        for (int c = 0; c < p.nZV; ++c) push(&tmZ, c * kChunk, kt * kTile, b);
      };
      push_qk(tiles[0]);
      for (int s = 0; s < nkt && ok; ++s) {
        if (s + 1 < nkt) push_qk(tiles[s + 1]);
        push_pv(tiles[s]);
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
      bool ok = mbar_wait(q_full, 0, wc, 2);
      tc_fence_after();
      int st = 0;
      uint32_t ph = 0;
      const uint32_t idS = idesc_f16(128, 128, 0, 0);
      const uint32_t idO = idesc_f16(128, 64, 0, 1);
      const uint32_t sQa = smem_u32(sQ), sRa = smem_u32(sRing);
      auto mma_qk = [&]() -> bool {
        // key chunks in ring order: the pair part first (each z2 chunk meets nqz
        // Qhat chunks: u hi, u lo), the head part (scalar and point columns)
        // last, so the small pair terms accumulate before the large point terms
        const int nb = p.nZ + p.nKH;
        for (int c = 0; c < nb; ++c) {
          if (!mbar_wait(&full[st], ph, wc, 3)) return false;
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
        return true;
      };
      auto mma_pv = [&](int s) -> bool {
        const int nchunk = p.nVH + p.nZV;
        for (int c = 0; c < nchunk; ++c) {
          if (!mbar_wait(&full[st], ph, wc, 4)) return false;
          tc_fence_after();
          const uint32_t b0 = sRa + st * kChunkBytes;
          const uint32_t dcol = tmem + (uint32_t)(p.tmemO + c * kChunk);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t bd = desc_mnmajor_sw128(b0 + kk * 2048, kChunkBytes);
            mma_ts(dcol, tmem + kTmemP + kk * 8, bd, idO, (s > 0 || kk > 0) ? 1u : 0u);
            if (SPLIT) mma_ts(dcol, tmem + kTmemP + 64 + kk * 8, bd, idO, 1u);
          }
          tc_commit(&empty[st]);
          if (++st == p.nst) { st = 0; ph ^= 1u; }
        }
        tc_commit(pv_done);
        return true;
      };
      if (ok) ok = mma_qk();
      for (int s = 0; ok && s < nkt; ++s) {
        if (s + 1 < nkt) {
          if (!mbar_wait(s_free, s & 1, wc, 5)) break;
          tc_fence_after();
          if (!mma_qk()) break;
        }
        if (!mbar_wait(p_full, s & 1, wc, 6)) break;
        tc_fence_after();
        if (!mma_pv(s)) break;
      }
      // every MMA this thread issued has finished before the CTA tears down
      tc_commit(drain);
      drain_wait(drain, 0, a.timeout_ns);
    }
  } else if (warp == 2 || warp == 3) {
    // ------------------------------------------------------------ per-key terms
    // kterm[s][j] = -g sum_p |b'_p|^2 + 2g D_sj . sum_p b'_p  (-inf for a masked or
    // absent key), D_sj = origin of query group s - origin of key j's group; the
    // four key-group origins of the tile go to shared memory as well.
    const int tt = threadIdx.x - 64;
    const float g = point_weight(load_raw(a, h), p.P);
    float4 oq[4];
#pragma unroll
    for (int sq = 0; sq < 4; ++sq) oq[sq] = a.orig[(size_t)b * p.nG + qt * 4 + sq];
    for (int s = 0; s < nkt; ++s) {
      const int kb = s & 1;
      const bool okw = mbar_wait(&kt_empty[kb], ((s >> 1) & 1) ^ 1, wc, 10);
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
    for (int s = 0; s < nkt; ++s) {
      const int kt = tiles[s];
      const int kb = s & 1;

      ok = mbar_wait(s_full, s & 1, wc, 7);
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

      ok = mbar_wait(&kt_full[kb], (s >> 1) & 1, wc, 11);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
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
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const float dd[3] = {oqs.x - okg[t].x, oqs.y - okg[t].y, oqs.z - okg[t].z};
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const float* kj = kpb + (t * 32 + e) * P3;
            float d2 = 0.f;
            for (int x = 0; x < P3; ++x) {
              const float d = (aq[x] + dd[x % 3]) - kj[x];
              d2 = fmaf(d, d, d2);
            }
            sv[t][e] = __float_as_uint(__uint_as_float(sv[t][e]) - g * d2);
          }
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
          rs0 += p0 + p1;
          rs1 += p2 + p3;
          const int w = (t & 1) * 16 + e / 2;
          pk[t >> 1][w] = pack_half2(p0, p1);
          pk[t >> 1][w + 1] = pack_half2(p2, p3);
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
      if (s > 0) {
        ok = mbar_wait(pv_done, (s - 1) & 1, wc, 8);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        tc_fence_after();
      }
      if (__any_sync(0xffffffffu, resc)) {
        const float f = resc ? alpha : 1.f;
        for (int c = 0; c < p.Ocols; c += 32) {
          uint32_t o[32];
          tmem_ld32(trow + (uint32_t)(p.tmemO + c), o);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * f);
          tmem_st32(trow + (uint32_t)(p.tmemO + c), o);
        }
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
    }
    if (ok && nkt > 0) {
      ok = mbar_wait(pv_done, (nkt - 1) & 1, wc, 9);
      ok = __all_sync(0xffffffffu, ok);
      tc_fence_after();
    }
    const float inv = l > 0.f ? 1.f / l : 0.f;
    if (ok && nkt > 0) {
      float* orow = a.O + (((size_t)b * N + i) * p.H + h) * p.Ocols;
      for (int c = 0; c < p.Ocols; c += 32) {
        uint32_t o[32];
        tmem_ld32(trow + (uint32_t)(p.tmemO + c), o);
        tmem_ld_wait();
        if (in_range) {
#pragma unroll
          for (int e = 0; e < 32; e += 4)
            *reinterpret_cast<float4*>(orow + c + e) =
                make_float4(__uint_as_float(o[e]) * inv, __uint_as_float(o[e + 1]) * inv,
                            __uint_as_float(o[e + 2]) * inv, __uint_as_float(o[e + 3]) * inv);
        }
      }
    }
    if (in_range) {
      a.W[((size_t)b * N + i) * p.H + h] = make_float4(Wx * inv, Wy * inv, Wz * inv, l);
      a.stats[(size_t)bh * N + i] = make_float2(M, l);
      if (a.lse != nullptr) a.lse[(size_t)bh * N + i] = l > 0.f ? (M + log2f(l)) * kLn2 + qv.w : -INFINITY;
    }
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

cudaError_t launch_core(const Plan& p, const Inputs& in, const Work& w, const Outputs& out,
                        const CUtensorMap& tmQ, const CUtensorMap& tmKH, const CUtensorMap& tmVH,
                        const CUtensorMap& tmZ, const DeviceCtl& ctl, cudaStream_t s) {
  CoreArgs a;
  a.p = p;
  a.kvec = w.kvec; a.qvec = w.qvec; a.QP = w.QP; a.KP = w.KP; a.orig = w.orig; a.flag = w.flag;
  a.mask = in.mask; a.pair_mask = in.pair_mask; a.raw = in.raw;
  a.O = w.O; a.W = w.W; a.stats = w.stats; a.lse = out.lse;
  a.status = ctl.status; a.timeout_ns = ctl.timeout_ns;
  dim3 grid(p.nT, p.H, p.B);
  if (p.f32) {
    auto kfn = fipa_core_kernel<true>;
    cudaError_t e = cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)p.core_smem);
    if (e != cudaSuccess) return e;
    kfn<<<grid, 256, p.core_smem, s>>>(tmQ, tmKH, tmVH, tmZ, a);
  } else {
    auto kfn = fipa_core_kernel<false>;
    cudaError_t e = cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)p.core_smem);
    if (e != cudaSuccess) return e;
    kfn<<<grid, 256, p.core_smem, s>>>(tmQ, tmKH, tmVH, tmZ, a);
  }
  return cudaGetLastError();
}

}  // namespace fipa
