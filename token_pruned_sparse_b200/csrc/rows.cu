// Row movement of the pruned path: KV-cache sync, output restoration, gather.
//
//   kv_sync      [HSA] 2.2 (2): fresh K/V of the active tokens overwrite their
//                rows of the per-layer cache; the other rows stay stale but valid.
//                Optional noise-aware duplication ([LIPAR] 2.C): pruned rows
//                enter attention as a*clean + b*fresh Gaussian noise.
//   scatter_out  [LIPAR] Dutch summary 2.D: pruned tokens are restored by
//                duplication, so the full-length output keeps their cached rows.
//   gather_rows  [HSA] 2.2 (1): only active tokens enter the QKV projection.
//
// All HBM-bound. One warp moves one row (H*d bf16 = 3..6 KB) at a time with
// 16-byte vector loads, several vectors in flight per lane, rows handed out
// grid-stride so every SM streams. Indices outside [0, N) are skipped and
// recorded in the device status word.
//
// Re-noise draws eps with Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel
// Random Numbers: As Easy as 1, 2, 3", SC'11) and the Box-Muller transform
// (Box & Muller, Ann. Math. Stat. 1958), generated where the row is written so
// the normals never touch memory.
#include "trace.cuh"
#include "tps_internal.cuh"
#include "warp_search.cuh"

namespace tps {
namespace {

constexpr int kUnroll = 4;
// Row moves and the re-noise pass run as 128-thread blocks, up to 16 per SM: at
// the HSA size rows move at 6.42 TB/s against 6.09-6.25 TB/s with 256-thread
// blocks and 8 per SM, and re-noise gains 2%.
constexpr int kMoveThreads = 128;
constexpr int kMoveWarps = kMoveThreads / 32;

// ---- row move: dst[dst_row] = src[src_row] for one or two tensors -----------------
// kScatter: dst row = idx[j], src row = j.  !kScatter: dst row = j, src row = idx[j].
template <bool kScatter>
__global__ void __launch_bounds__(kMoveThreads) rows_move(uint4* __restrict__ d0, const uint4* __restrict__ s0,
                                                      uint4* __restrict__ d1, const uint4* __restrict__ s1,
                                                      const int32_t* __restrict__ idx,
                                                      const int32_t* __restrict__ count, int64_t cap,
                                                      int64_t N, int vpr, unsigned int* status) {
  const int lane = threadIdx.x & 31;
  const int64_t rows = active_count(count, cap);
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * kMoveThreads + threadIdx.x) >> 5;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * kMoveWarps;
  for (int64_t j = warp; j < rows; j += nwarps) {
    const int64_t n = idx[j];
    if (n < 0 || n >= N) {
      if (lane == 0) raise_status(status, STATUS_BOUNDS);
      continue;
    }
    const int64_t srow = (kScatter ? j : n) * vpr;
    const int64_t drow = (kScatter ? n : j) * vpr;
    for (int v0 = lane; v0 < vpr; v0 += 32 * kUnroll) {
      uint4 a[kUnroll], b[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int v = v0 + u * 32;
        if (v < vpr) {
          a[u] = s0[srow + v];
          if (s1) b[u] = s1[srow + v];
        }
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int v = v0 + u * 32;
        if (v < vpr) {
          d0[drow + v] = a[u];
          if (d1) d1[drow + v] = b[u];
        }
      }
    }
  }
}

// ---- Philox4x32-10 and Box-Muller ------------------------------------------------
constexpr uint32_t kM0 = 0xD2511F53u, kM1 = 0xCD9E8D57u;  // round multipliers
constexpr uint32_t kW0 = 0x9E3779B9u, kW1 = 0xBB67AE85u;  // Weyl key increments

// The key of round r is (k0 + r*W0, k1 + r*W1) mod 2^32. The schedule is computed
// once on the host and passed as a __grid_constant__ kernel parameter, so each
// round reads its key straight from the constant bank as an operand of the XOR.
struct PhiloxKeys {
  uint32_t k0[10];
  uint32_t k1[10];
};

inline PhiloxKeys philox_keys(uint64_t seed) {
  PhiloxKeys K;
  uint32_t k0 = static_cast<uint32_t>(seed), k1 = static_cast<uint32_t>(seed >> 32);
  for (int r = 0; r < 10; ++r) {
    K.k0[r] = k0;
    K.k1[r] = k1;
    k0 += kW0;
    k1 += kW1;
  }
  return K;
}

__device__ __forceinline__ uint4 philox10(uint4 c, const PhiloxKeys& K) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    const uint32_t hi0 = __umulhi(kM0, c.x), lo0 = kM0 * c.x;
    const uint32_t hi1 = __umulhi(kM1, c.z), lo1 = kM1 * c.z;
    c = make_uint4(hi1 ^ c.y ^ K.k0[r], lo1, hi0 ^ c.w ^ K.k1[r], lo0);
  }
  return c;
}

// u = (floor(w / 2^9) + 1/2) * 2^-23: exact in fp32, strictly inside (0, 1).
// Built from the bits: 1 + k * 2^-23 (exponent of 1.0, mantissa k = w >> 9),
// minus (1 - 2^-24); both operands and the difference are exact in fp32.
__device__ __forceinline__ float uniform01(uint32_t w) {
  return __uint_as_float(0x3F800000u | (w >> 9)) - 0.99999994039535522461f;
}

__device__ __forceinline__ float sqrt_approx(float x) {
  float y;
  asm("sqrt.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Box-Muller on one word pair: z0 = r cos(2 pi ub), z1 = r sin(2 pi ub),
// r = sqrt(-2 ln ua). The angle is taken as 2 pi (ub - 1/2) in (-pi, pi), where
// the hardware sine/cosine are accurate, and the signs folded back.
// -2 ln u for u in (0, 1): the hardware base-2 logarithm times -2 ln 2, except
// for u > 0.995 (t = 1 - u < 0.005, exact in fp32), where the Taylor series of
// -2 ln(1 - t) = 2t (1 + t/2 + t^2/3 + ...) to the t^2 term is accurate to t^3/4.
__device__ __forceinline__ float neg2ln(float u) {
  float l2;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(l2) : "f"(u));
  const float t = 1.0f - u;
  const float ser = 2.0f * t * fmaf(t, fmaf(t, 0.333333343f, 0.5f), 1.0f);
  return t < 0.005f ? ser : -1.38629436111989061883f * l2;
}

__device__ __forceinline__ void box_muller(uint32_t wa, uint32_t wb, float& z0, float& z1) {
  const float ua = uniform01(wa), ub = uniform01(wb);
  const float r = sqrt_approx(neg2ln(ua));         // hardware sqrt, ~2^-23 relative
  // 2 pi (ub - 1/2) in one rounding: 2 pi and pi are exact doubles of each other in fp32
  const float th = fmaf(6.28318530717958647692f, ub, -3.14159265358979323846f);
  float sn, cs;
  __sincosf(th, &sn, &cs);
  z0 = -r * cs;
  z1 = -r * sn;
}

// Eight normals for the flat elements e0 .. e0+7 (e0 % 8 == 0) of tensor t.
__device__ __forceinline__ void normals8(uint64_t e0, uint32_t step, uint32_t t, const PhiloxKeys& K,
                                         float z[8]) {
  const uint64_t q = e0 >> 2;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint64_t qq = q + h;
    const uint4 w = philox10(make_uint4(static_cast<uint32_t>(qq), static_cast<uint32_t>(qq >> 32), step, t), K);
    box_muller(w.x, w.y, z[4 * h + 0], z[4 * h + 1]);
    box_muller(w.z, w.w, z[4 * h + 2], z[4 * h + 3]);
  }
}

__device__ __forceinline__ uint4 renoise_vec(uint4 c, float a, float b, const float z[8]) {
  const uint32_t cw[4] = {c.x, c.y, c.z, c.w};
  const float2 a2 = make_float2(a, a), b2 = make_float2(b, b);
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    // a*x, then b*z + (a*x): the same two roundings per element as fmaf(b, z, a * x)
    const float2 r = __ffma2_rn(b2, make_float2(z[2 * i], z[2 * i + 1]),
                                __fmul2_rn(a2, make_float2(bf16lo(cw[i]), bf16hi(cw[i]))));
    o[i] = pack_bf16x2(r.x, r.y);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// ---- kv_sync with re-noise: one pass over all N rows --------------------------------
// A warp owns a run of kRun consecutive rows; one warp-cooperative search finds the first
// active index >= the run start, then the (ascending) list is walked in step.
constexpr int kRun = 8;
// Ten resident blocks per SM (at most 48 registers; a few bytes spill) against
// eight at the compiler's 59 registers: the memory stream has more rows in
// flight and the pass runs 2.7% faster at the HSA size (0.615 -> 0.599 ms).
constexpr int kRenoiseBlocks = 10;

__global__ void __launch_bounds__(kMoveThreads, kRenoiseBlocks) kv_sync_renoise(
    uint4* __restrict__ kc, uint4* __restrict__ vc, const uint4* __restrict__ kf,
    const uint4* __restrict__ vf, const int32_t* __restrict__ idx, const int32_t* __restrict__ count,
    int64_t cap, int64_t N, int vpr, float a, float b, const __grid_constant__ PhiloxKeys keys, uint32_t step,
    uint4* __restrict__ ke, uint4* __restrict__ ve, unsigned int* status) {
  const int lane = threadIdx.x & 31;
  const int64_t cnt = active_count(count, cap);
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * kMoveThreads + threadIdx.x) >> 5;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * kMoveWarps;
  const int64_t nruns = (N + kRun - 1) / kRun;
  const uint64_t epr = static_cast<uint64_t>(vpr) * 8;  // elements per row
  for (int64_t run = warp; run < nruns; run += nwarps) {
    const int64_t r0 = run * kRun;
    int64_t p = warp_lower_bound(idx, cnt, r0, lane);   // first list entry >= r0
    for (int64_t n = r0; n < r0 + kRun && n < N; ++n) {
      const bool active = p < cnt && idx[p] == n;
      const int64_t row = n * vpr;
      if (active) {
        const int64_t frow = p * vpr;
        for (int v = lane; v < vpr; v += 32) {
          const uint4 x = kf[frow + v];
          const uint4 y = vf[frow + v];
          kc[row + v] = x;
          ke[row + v] = x;
          vc[row + v] = y;
          ve[row + v] = y;
        }
        ++p;
      } else {
        uint4 x = make_uint4(0u, 0u, 0u, 0u), y = x;
        if (lane < vpr) {
          x = kc[row + lane];
          y = vc[row + lane];
        }
        for (int v = lane; v < vpr; v += 32) {
          uint4 xn = x, yn = y;
          if (v + 32 < vpr) {                       // the next vector's loads overlap this one's math
            xn = kc[row + v + 32];
            yn = vc[row + v + 32];
          }
          const uint64_t e0 = static_cast<uint64_t>(n) * epr + static_cast<uint64_t>(v) * 8;
          float z[8];
          normals8(e0, step, 0u, keys, z);
          ke[row + v] = renoise_vec(x, a, b, z);
          normals8(e0, step, 1u, keys, z);
          ve[row + v] = renoise_vec(y, a, b, z);
          x = xn;
          y = yn;
        }
      }
    }
    // entries of idx inside this run that are not strictly ascending, or
    // outside [0, N), were not consumed: flag them
    if (lane == 0) {
      const int64_t end = r0 + kRun < N ? r0 + kRun : N;
      if (p < cnt && idx[p] < end) raise_status(status, STATUS_BOUNDS);
      if (run == nruns - 1 && cnt > 0 && (idx[cnt - 1] >= N || idx[0] < 0)) raise_status(status, STATUS_BOUNDS);
    }
  }
}

__global__ void philox_fill(uint4* out, uint64_t q0, int64_t nq, const __grid_constant__ PhiloxKeys keys,
                            uint32_t step, uint32_t t) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < nq; i += stride) {
    const uint64_t q = q0 + static_cast<uint64_t>(i);
    out[i] = philox10(make_uint4(static_cast<uint32_t>(q), static_cast<uint32_t>(q >> 32), step, t), keys);
  }
}

unsigned int move_grid(int64_t rows) {
  int64_t g = (rows + kMoveWarps - 1) / kMoveWarps;
  const int64_t cap = static_cast<int64_t>(sm_count()) * 16;
  if (g > cap) g = cap;
  if (g < 1) g = 1;
  return static_cast<unsigned int>(g);
}

int check_rows(const char* who, int64_t cap, int64_t N, int H, int d) {
  if (cap < 0 || N < 1 || N >= (INT64_C(1) << 31))
    return fail(TPS_ERR_SHAPE, "%s: need cap >= 0 and 1 <= N < 2^31 (cap=%lld N=%lld)", who, (long long)cap, (long long)N);
  if (d != 64 && d != 128) return fail(TPS_ERR_INVALID_ARG, "%s: d=%d must be 64 or 128", who, d);
  if (H < 1 || static_cast<int64_t>(H) * d > 16384)
    return fail(TPS_ERR_SHAPE, "%s: H=%d must satisfy 1 <= H*d <= 16384", who, H);
  return TPS_OK;
}

}  // namespace
}  // namespace tps

using namespace tps;

extern "C" int tps_gather_rows(void* dst, const void* src, const int32_t* idx, const int32_t* count,
                               int64_t cap, int64_t N, int64_t row_bytes, tps_stream stream) {
  TPS_TRACE("tps_gather_rows");
  if (!dst || !src || !idx || !count) return fail(TPS_ERR_INVALID_ARG, "tps_gather_rows: null pointer");
  if (cap < 0 || N < 1 || N >= (INT64_C(1) << 31)) return fail(TPS_ERR_SHAPE, "tps_gather_rows: bad cap/N");
  if (row_bytes < 16 || row_bytes % 16 || row_bytes > (INT64_C(1) << 20))
    return fail(TPS_ERR_SHAPE, "tps_gather_rows: row_bytes=%lld must be a multiple of 16 in [16, 1 MiB]", (long long)row_bytes);
  if (!aligned16(dst) || !aligned16(src)) return fail(TPS_ERR_ALIGN, "tps_gather_rows: rows must be 16-byte aligned");
  int err;
  unsigned int* st = device_status(&err);
  if (!st) return err;
  if (cap == 0) return ok();
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  rows_move<false><<<move_grid(cap), kMoveThreads, 0, s>>>(static_cast<uint4*>(dst), static_cast<const uint4*>(src),
                                                      nullptr, nullptr, idx, count, cap, N,
                                                      static_cast<int>(row_bytes / 16), st);
  if (int e = launch_status("tps_gather_rows")) return e;
  return ok();
}

extern "C" int scatter_out(tps_bf16* o_full, const tps_bf16* o_act, const int32_t* idx,
                           const int32_t* count, int64_t cap, int64_t N, int H, int d,
                           tps_stream stream) {
  TPS_TRACE("scatter_out");
  if (!o_full || !o_act || !idx || !count) return fail(TPS_ERR_INVALID_ARG, "scatter_out: null pointer");
  if (int e = check_rows("scatter_out", cap, N, H, d)) return e;
  if (!aligned16(o_full) || !aligned16(o_act)) return fail(TPS_ERR_ALIGN, "scatter_out: rows must be 16-byte aligned");
  int err;
  unsigned int* st = device_status(&err);
  if (!st) return err;
  if (cap == 0) return ok();
  const int vpr = H * d / 8;
  rows_move<true><<<move_grid(cap), kMoveThreads, 0, static_cast<cudaStream_t>(stream)>>>(
      reinterpret_cast<uint4*>(o_full), reinterpret_cast<const uint4*>(o_act), nullptr, nullptr, idx,
      count, cap, N, vpr, st);
  if (int e = launch_status("scatter_out")) return e;
  return ok();
}

extern "C" int kv_sync(tps_bf16* k_cache, tps_bf16* v_cache, const tps_bf16* k_fresh,
                       const tps_bf16* v_fresh, const int32_t* idx, const int32_t* count, int64_t cap,
                       int64_t N, int H, int d, const tps_renoise* rn, tps_bf16* k_eff,
                       tps_bf16* v_eff, tps_stream stream) {
  TPS_TRACE("kv_sync");
  if (!k_cache || !v_cache || !k_fresh || !v_fresh || !idx || !count)
    return fail(TPS_ERR_INVALID_ARG, "kv_sync: null pointer");
  if (int e = check_rows("kv_sync", cap, N, H, d)) return e;
  if (rn && (!k_eff || !v_eff)) return fail(TPS_ERR_INVALID_ARG, "kv_sync: re-noise needs k_eff and v_eff");
  if (!aligned16(k_cache) || !aligned16(v_cache) || !aligned16(k_fresh) || !aligned16(v_fresh) ||
      (rn && (!aligned16(k_eff) || !aligned16(v_eff))))
    return fail(TPS_ERR_ALIGN, "kv_sync: rows must be 16-byte aligned");
  int err;
  unsigned int* st = device_status(&err);
  if (!st) return err;
  const int vpr = H * d / 8;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (!rn) {
    if (cap == 0) return ok();
    rows_move<true><<<move_grid(cap), kMoveThreads, 0, s>>>(
        reinterpret_cast<uint4*>(k_cache), reinterpret_cast<const uint4*>(k_fresh),
        reinterpret_cast<uint4*>(v_cache), reinterpret_cast<const uint4*>(v_fresh), idx, count, cap, N,
        vpr, st);
  } else {
    const int64_t runs = (N + kRun - 1) / kRun;
    kv_sync_renoise<<<move_grid(runs), kMoveThreads, 0, s>>>(
        reinterpret_cast<uint4*>(k_cache), reinterpret_cast<uint4*>(v_cache),
        reinterpret_cast<const uint4*>(k_fresh), reinterpret_cast<const uint4*>(v_fresh), idx, count, cap,
        N, vpr, rn->a, rn->b, philox_keys(rn->seed), rn->step, reinterpret_cast<uint4*>(k_eff),
        reinterpret_cast<uint4*>(v_eff), st);
  }
  if (int e = launch_status("kv_sync")) return e;
  return ok();
}

extern "C" int tps_philox_fill(uint32_t* out, uint64_t q0, int64_t nq, uint64_t seed, uint32_t step,
                               uint32_t tensor, tps_stream stream) {
  TPS_TRACE("tps_philox_fill");
  if (!out) return fail(TPS_ERR_INVALID_ARG, "tps_philox_fill: out is null");
  if (nq < 0) return fail(TPS_ERR_SHAPE, "tps_philox_fill: nq < 0");
  if (!aligned16(out)) return fail(TPS_ERR_ALIGN, "tps_philox_fill: out must be 16-byte aligned");
  if (nq == 0) return ok();
  int64_t g = (nq + 255) / 256;
  if (g > 4096) g = 4096;
  philox_fill<<<static_cast<unsigned int>(g), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      reinterpret_cast<uint4*>(out), q0, nq, philox_keys(seed), step, tensor);
  if (int e = launch_status("tps_philox_fill")) return e;
  return ok();
}
