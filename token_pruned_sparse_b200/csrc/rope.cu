// kv_rerotate: keys of pruned tokens reused from the previous frame, moved to
// their own rotary position.
//
// [LIPAR] "Training-free Latent Inter-Frame Pruning with Attention Recovery",
// Dutch summary 2.C (M-degree approximation): the K/V of a pruned token are
// approximated by the cached K/V of the previous frame, taking the RoPE
// rotations into account. [TR] "Timeripple", Metodologia 1: the rotary
// channels of a head form temporal, x and y groups.
//
// Reading: a head's d channels are the groups [t | x | y] of sizes dims[0..2];
// inside group a the adjacent channels (o_a + 2j, o_a + 2j + 1) are pair j
// with frequency base^(-2j / d_a). A cached key of a pruned token moves by the
// offset shift = (s_t, s_x, s_y): pair j turns by phi = s_a * base^(-2j/d_a),
// (x, y) -> (x cos phi - y sin phi, x sin phi + y cos phi). Active rows are
// copied unchanged (after kv_sync they hold the fresh keys).
//
// One pass over the N rows, HBM-bound (2 * H * d * 2 bytes per row): a warp
// owns a run of consecutive rows, finds the first active index of the run with
// one warp-cooperative search and walks the ascending list in step. The
// (cos, sin) table of the d/2 pairs is computed on the host in double
// precision, rounded to fp32 and staged in shared memory.
#include <cmath>

#include "trace.cuh"
#include "tps_internal.cuh"
#include "warp_search.cuh"

namespace tps {
namespace {

constexpr int kThreads = 128;
constexpr int kWarps = kThreads / 32;
constexpr int kRun = 8;
constexpr int kUnroll = 4;      // 16-byte vectors per lane in flight
constexpr int kMaxPairs = 64;   // d <= 128

struct RopeTable {
  float2 cs[kMaxPairs];   // (cos phi, sin phi) of channel pair p = c / 2
};

__device__ __forceinline__ uint32_t rotate_pair(uint32_t w, float2 cs) {
  const float x = bf16lo(w), y = bf16hi(w);
  return pack_bf16x2(fmaf(x, cs.x, -y * cs.y), fmaf(x, cs.y, y * cs.x));
}

__global__ void __launch_bounds__(kThreads) rerotate_kernel(const uint4* k_cache, uint4* k_eff,
                                                          const int32_t* __restrict__ idx,
                                                          const int32_t* __restrict__ count, int64_t cap,
                                                          int64_t N, int vpr, int vph,
                                                          const __grid_constant__ RopeTable tab,
                                                          unsigned int* status) {
  __shared__ __align__(16) float2 s_cs[kMaxPairs];
  if (threadIdx.x < kMaxPairs) s_cs[threadIdx.x] = tab.cs[threadIdx.x];
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int64_t cnt = active_count(count, cap);
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x) >> 5;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * kWarps;
  const int64_t nruns = (N + kRun - 1) / kRun;
  for (int64_t run = warp; run < nruns; run += nwarps) {
    const int64_t r0 = run * kRun;
    int64_t p = warp_lower_bound(idx, cnt, r0, lane);
    for (int64_t n = r0; n < r0 + kRun && n < N; ++n) {
      const bool active = p < cnt && idx[p] == n;
      const int64_t row = n * vpr;
      // kUnroll vectors per lane in flight before any is used
      for (int v0 = lane; v0 < vpr; v0 += 32 * kUnroll) {
        uint4 x[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u)
          if (v0 + 32 * u < vpr) x[u] = k_cache[row + v0 + 32 * u];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
          const int v = v0 + 32 * u;
          if (v >= vpr) continue;
          if (active) {
            k_eff[row + v] = x[u];
          } else {
            const int p0 = (v % vph) * 4;                  // first channel pair of this vector
            const float4 c01 = *reinterpret_cast<const float4*>(&s_cs[p0]);
            const float4 c23 = *reinterpret_cast<const float4*>(&s_cs[p0 + 2]);
            k_eff[row + v] = make_uint4(rotate_pair(x[u].x, make_float2(c01.x, c01.y)),
                                        rotate_pair(x[u].y, make_float2(c01.z, c01.w)),
                                        rotate_pair(x[u].z, make_float2(c23.x, c23.y)),
                                        rotate_pair(x[u].w, make_float2(c23.z, c23.w)));
          }
        }
      }
      if (active) ++p;
    }
    if (lane == 0) {
      const int64_t end = r0 + kRun < N ? r0 + kRun : N;
      if (p < cnt && idx[p] < end) raise_status(status, STATUS_BOUNDS);
      if (run == nruns - 1 && cnt > 0 && (idx[cnt - 1] >= N || idx[0] < 0)) raise_status(status, STATUS_BOUNDS);
    }
  }
}

}  // namespace
}  // namespace tps

using namespace tps;

extern "C" int kv_rerotate(const tps_bf16* k_cache, const int32_t* idx, const int32_t* count, int64_t cap,
                           int64_t N, int H, int d, const tps_rope* rope, tps_bf16* k_eff, tps_stream stream) {
  TPS_TRACE("kv_rerotate");
  if (!k_cache || !idx || !count || !rope || !k_eff) return fail(TPS_ERR_INVALID_ARG, "kv_rerotate: null pointer");
  if (cap < 0 || N < 1 || N >= (INT64_C(1) << 31))
    return fail(TPS_ERR_SHAPE, "kv_rerotate: need cap >= 0 and 1 <= N < 2^31");
  if (d != 64 && d != 128) return fail(TPS_ERR_INVALID_ARG, "kv_rerotate: d=%d must be 64 or 128", d);
  if (H < 1 || static_cast<int64_t>(H) * d > 16384)
    return fail(TPS_ERR_SHAPE, "kv_rerotate: H=%d must satisfy 1 <= H*d <= 16384", H);
  int sum = 0;
  for (int a = 0; a < 3; ++a) {
    if (rope->dims[a] < 0 || rope->dims[a] % 2)
      return fail(TPS_ERR_INVALID_ARG, "kv_rerotate: group %d has %d channels (must be even and >= 0)", a,
                  rope->dims[a]);
    if (rope->shift[a] < -(1 << 20) || rope->shift[a] > (1 << 20))
      return fail(TPS_ERR_INVALID_ARG, "kv_rerotate: |shift| must be <= 2^20");
    sum += rope->dims[a];
  }
  if (sum != d) return fail(TPS_ERR_INVALID_ARG, "kv_rerotate: groups sum to %d channels, d=%d", sum, d);
  if (!(rope->base > 0.f) || !std::isfinite(rope->base))
    return fail(TPS_ERR_INVALID_ARG, "kv_rerotate: base must be finite and > 0");
  if (!aligned16(k_cache) || !aligned16(k_eff)) return fail(TPS_ERR_ALIGN, "kv_rerotate: rows must be 16-byte aligned");
  RopeTable tab{};
  int pr = 0;
  for (int a = 0; a < 3; ++a) {
    const int da = rope->dims[a];
    for (int j = 0; j < da / 2; ++j, ++pr) {
      const double phi = static_cast<double>(rope->shift[a]) *
                         std::pow(static_cast<double>(rope->base), -2.0 * j / static_cast<double>(da));
      tab.cs[pr] = make_float2(static_cast<float>(std::cos(phi)), static_cast<float>(std::sin(phi)));
    }
  }
  int err;
  unsigned int* st = device_status(&err);
  if (!st) return err;
  const int vpr = H * d / 8;
  const int64_t runs = (N + kRun - 1) / kRun;
  int64_t g = (runs + kWarps - 1) / kWarps;
  const int64_t gmax = static_cast<int64_t>(sm_count()) * 16;
  g = g > gmax ? gmax : (g < 1 ? 1 : g);
  rerotate_kernel<<<static_cast<unsigned int>(g), kThreads, 0, static_cast<cudaStream_t>(stream)>>>(
      reinterpret_cast<const uint4*>(k_cache), reinterpret_cast<uint4*>(k_eff), idx, count, cap, N, vpr, d / 8, tab,
      st);
  if (int e = launch_status("kv_rerotate")) return e;
  return ok();
}
