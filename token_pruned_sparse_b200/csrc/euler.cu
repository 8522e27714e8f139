// hsa_euler_update: the cached Euler update of HSA.
//
// [HSA] "Asignacion de Pasos Heterogenea", 2.3: every token keeps the velocity
// predicted at its most recent active step; at each global step all N tokens
// advance by the same Euler increment (sigma_{i+1} - sigma_i) -- active tokens
// with the velocity just computed, skipped tokens with their cached one -- in
// one branch-free operation over the whole sequence.
//
// Fused, HBM-bound single pass: the velocity cache is refreshed for the active
// rows and every row of the fp32 state advances, v read once per token. A warp
// owns a group of 4 runs of 8 consecutive tokens: one warp-cooperative search in
// the ascending index list finds the group's first active entry, and each run
// continues from where the previous one stopped. Per run a warp-wide OR builds
// the run's active mask, and the warp then sweeps the run's (token, 16-byte
// vector) items with several loads in flight per lane.
#include "trace.cuh"
#include "tps_internal.cuh"
#include "warp_search.cuh"

namespace tps {
namespace {

constexpr int kThreads = 128;
constexpr int kWarps = kThreads / 32;
constexpr int kRun = 8;

// kVpr > 0: 16-byte velocity vectors per row fixed at compile time, so a lane's
// items of a run are fully unrolled and their loads issued together.
template <int kVpr>
__global__ void __launch_bounds__(kThreads) euler_kernel(float* __restrict__ x, uint4* __restrict__ vcache,
                                                         const uint4* __restrict__ vfresh,
                                                         const int32_t* __restrict__ idx,
                                                         const int32_t* __restrict__ count, int64_t cap, int64_t N,
                                                         int vpr_rt, float dsigma, unsigned int* status) {
  const int vpr = kVpr > 0 ? kVpr : vpr_rt;
  const int lane = threadIdx.x & 31;
  const int64_t cnt = active_count(count, cap);
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x) >> 5;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * kWarps;
  const int64_t nruns = (N + kRun - 1) / kRun;
  const int items = kRun * vpr;                 // (token, vector) pairs of one run
  constexpr int kGroup = 4;                     // runs per search: later runs continue from the last
  const int64_t ngroups = (nruns + kGroup - 1) / kGroup;
  for (int64_t grp = warp; grp < ngroups; grp += nwarps) {
    int64_t lo = warp_lower_bound(idx, cnt, grp * kGroup * kRun, lane);   // first list entry >= the group start
    for (int64_t run = grp * kGroup; run < nruns && run < (grp + 1) * kGroup; ++run) {
      const int64_t r0 = run * kRun;
      // lanes 0..7 look at the next 8 list entries; those below r0 + 8 are active rows of this run
      const int64_t mine = (lane < kRun && lo + lane < cnt) ? idx[lo + lane] : INT64_MAX;
      const bool in_run = mine >= r0 && mine < r0 + kRun;
      const unsigned int rowbits =
          __reduce_or_sync(0xffffffffu, in_run ? (1u << static_cast<unsigned int>(mine - r0)) : 0u);
      const unsigned int nin = __popc(__ballot_sync(0xffffffffu, in_run));
      if (lane == 0) {
        // duplicates in the list, or entries outside [0, N), are not consumed
        if (nin != static_cast<unsigned int>(__popc(rowbits))) raise_status(status, STATUS_BOUNDS);
        if (run == nruns - 1 && cnt > 0 && (idx[cnt - 1] >= N || idx[0] < 0)) raise_status(status, STATUS_BOUNDS);
      }
#pragma unroll
      for (int i = lane; i < (kVpr > 0 ? kRun * kVpr : items); i += 32) {
        const int r = i / vpr, v = i - r * vpr;
        const int64_t n = r0 + r;
        if (n >= N) continue;
        uint4 vel;
        if ((rowbits >> r) & 1u) {
          const int64_t pos = lo + __popc(rowbits & ((1u << r) - 1u));
          vel = vfresh[pos * vpr + v];
          vcache[n * vpr + v] = vel;
        } else {
          vel = vcache[n * vpr + v];
        }
        float4* xp = reinterpret_cast<float4*>(x + (n * vpr + v) * 8);
        float4 x0 = xp[0], x1 = xp[1];
        x0.x = fmaf(dsigma, bf16lo(vel.x), x0.x);
        x0.y = fmaf(dsigma, bf16hi(vel.x), x0.y);
        x0.z = fmaf(dsigma, bf16lo(vel.y), x0.z);
        x0.w = fmaf(dsigma, bf16hi(vel.y), x0.w);
        x1.x = fmaf(dsigma, bf16lo(vel.z), x1.x);
        x1.y = fmaf(dsigma, bf16hi(vel.z), x1.y);
        x1.z = fmaf(dsigma, bf16lo(vel.w), x1.z);
        x1.w = fmaf(dsigma, bf16hi(vel.w), x1.w);
        xp[0] = x0;
        xp[1] = x1;
      }
      lo += nin;                                   // the next run's entries start after this run's
    }
  }
}

}  // namespace
}  // namespace tps

extern "C" int hsa_euler_update(float* x, tps_bf16* v_cache, const tps_bf16* v_fresh, const int32_t* idx,
                                const int32_t* count, int64_t cap, int64_t N, int64_t C, float dsigma,
                                tps_stream stream) {
  TPS_TRACE("hsa_euler_update");
  using namespace tps;
  if (!x || !v_cache || !idx || !count || (cap > 0 && !v_fresh))
    return fail(TPS_ERR_INVALID_ARG, "hsa_euler_update: null pointer");
  if (N < 1 || N >= (INT64_C(1) << 31) || cap < 0) return fail(TPS_ERR_SHAPE, "hsa_euler_update: need 1 <= N < 2^31, cap >= 0");
  if (C < 8 || C % 8 || C > 4096) return fail(TPS_ERR_SHAPE, "hsa_euler_update: C=%lld must be a multiple of 8 in [8, 4096]", (long long)C);
  if (!(dsigma == dsigma) || dsigma == INFINITY || dsigma == -INFINITY)
    return fail(TPS_ERR_INVALID_ARG, "hsa_euler_update: dsigma must be finite");
  if (!aligned16(x) || !aligned16(v_cache) || (v_fresh && !aligned16(v_fresh)))
    return fail(TPS_ERR_ALIGN, "hsa_euler_update: x, v_cache, v_fresh must be 16-byte aligned");
  int err;
  unsigned int* st = device_status(&err);
  if (!st) return err;
  const int64_t runs = ((N + kRun - 1) / kRun + 4 - 1) / 4;   // groups of runs
  int64_t grid = (runs + kWarps - 1) / kWarps;
  const int64_t maxg = static_cast<int64_t>(sm_count()) * 16;
  if (grid > maxg) grid = maxg;
  const dim3 g(static_cast<unsigned int>(grid));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint4* vc = reinterpret_cast<uint4*>(v_cache);
  const uint4* vf = reinterpret_cast<const uint4*>(v_fresh);
  const int vpr = static_cast<int>(C / 8);
  if (vpr == 16) euler_kernel<16><<<g, kThreads, 0, s>>>(x, vc, vf, idx, count, cap, N, vpr, dsigma, st);
  else if (vpr == 8) euler_kernel<8><<<g, kThreads, 0, s>>>(x, vc, vf, idx, count, cap, N, vpr, dsigma, st);
  else euler_kernel<0><<<g, kThreads, 0, s>>>(x, vc, vf, idx, count, cap, N, vpr, dsigma, st);
  if (int e = launch_status("hsa_euler_update")) return e;
  return ok();
}
