// lipar_score: relative-L1 change per latent token.
//
// [LIPAR] "Training-free Latent Inter-Frame Pruning with Attention Recovery",
// 2.B: a latent patch is compared, by L1 norm, with the patch at the same
// spatial location in the previous frame. [HSA] "Asignacion de Pasos
// Heterogenea", 2.1: tokens are grouped by the per-token relative L1 change of
// consecutive velocity predictions. Both reduce to
//     s = sum_c |cur_c - ref_c| / sum_c |ref_c|.
//
// HBM-bound: each token row (C bf16) is read with 16-byte vector loads by a
// group of L lanes and reduced with xor shuffles. In inter-frame mode the
// reference row of token (f,p) is the current row of token (f-1,p), one frame
// (HW rows) earlier; it was read moments before by another warp, so the second
// read is served by the 126 MB L2 and DRAM sees each latent once.
#include <cmath>

#include "trace.cuh"
#include "tps_internal.cuh"

namespace tps {
namespace {

// kV > 0: vectors per row known at compile time (all loads of an iteration are
// issued before any is used); kV == 0: runtime C. kG token groups per lane and
// iteration, spaced a grid stride apart, so more 16-byte loads are in flight per
// lane; the grid is one resident wave. (kG = 4 measured slower than 2 at the
// HSA size: fewer, longer-running warps.)
template <int L, int kV, int kG>
__global__ void __launch_bounds__(256) score_kernel(const uint16_t* __restrict__ x,
                                                    const uint16_t* __restrict__ xref,
                                                    const uint16_t* __restrict__ xprev,
                                                    int64_t HW, int Crt, int64_t N,
                                                    float* __restrict__ score) {
  constexpr int kTokPerWarp = 32 / L;
  const int lane = threadIdx.x & 31;
  const int sub = lane & (L - 1);
  const int V = kV > 0 ? kV : (Crt >> 3);  // 16-byte vectors per row
  const int C = kV > 0 ? kV * 8 : Crt;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const int64_t stride = nwarps * kTokPerWarp;
  for (int64_t w0 = warp * kTokPerWarp; w0 < N; w0 += kG * stride) {
    const uint16_t* cur[kG];
    const uint16_t* ref[kG];
    int64_t tt[kG];
    bool valid[kG];
#pragma unroll
    for (int k = 0; k < kG; ++k) {
      const int64_t t = w0 + k * stride + lane / L;
      tt[k] = t;
      valid[k] = t < N;
      ref[k] = nullptr;
      cur[k] = x + (valid[k] ? t : 0) * C;
      if (valid[k]) {
        if (xref) ref[k] = xref + t * C;
        else if (t >= HW) ref[k] = x + (t - HW) * C;
        else if (xprev) ref[k] = xprev + t * C;
      }
    }
    float num[kG], den[kG];
#pragma unroll
    for (int k = 0; k < kG; ++k) num[k] = 0.f, den[k] = 0.f;
#pragma unroll
    for (int v = sub; v < (kV > 0 ? kV : V); v += L) {
      uint4 a[kG], b[kG];
#pragma unroll
      for (int k = 0; k < kG; ++k)
        if (ref[k]) {
          a[k] = ld16(cur[k] + v * 8);
          b[k] = ld16(ref[k] + v * 8);
        }
#pragma unroll
      for (int k = 0; k < kG; ++k)
        if (ref[k]) {
          const uint32_t aw[4] = {a[k].x, a[k].y, a[k].z, a[k].w};
          const uint32_t bw[4] = {b[k].x, b[k].y, b[k].z, b[k].w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float c0 = bf16lo(aw[i]), c1 = bf16hi(aw[i]);
            const float r0 = bf16lo(bw[i]), r1 = bf16hi(bw[i]);
            num[k] += fabsf(c0 - r0) + fabsf(c1 - r1);
            den[k] += fabsf(r0) + fabsf(r1);
          }
        }
    }
#pragma unroll
    for (int k = 0; k < kG; ++k) {
#pragma unroll
      for (int o = L / 2; o > 0; o >>= 1) {
        num[k] += __shfl_xor_sync(0xffffffffu, num[k], o);
        den[k] += __shfl_xor_sync(0xffffffffu, den[k], o);
      }
      if (valid[k] && sub == 0) {
        float s;
        if (!ref[k]) s = INFINITY;                  // frame 0 without a predecessor
        else if (den[k] > 0.f) s = num[k] / den[k];
        else s = num[k] > 0.f ? INFINITY : 0.f;
        score[tt[k]] = s;
      }
    }
  }
}

template <int L, int kV, int kG>
void launch_score(const uint16_t* x, const uint16_t* xr, const uint16_t* xp, int64_t HW, int C,
                  int64_t N, float* score, cudaStream_t st) {
  constexpr int kThreads = 256;
  const int64_t tok_per_block = (kThreads / 32) * (32 / L);
  int64_t blocks = (N + kG * tok_per_block - 1) / (kG * tok_per_block);
  static std::atomic<int> per_sm[64];           // resident blocks per SM (one wave), per device
  int dev = 0;
  cudaGetDevice(&dev);
  int b = dev >= 0 && dev < 64 ? per_sm[dev].load(std::memory_order_relaxed) : 0;
  if (!b) {
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, score_kernel<L, kV, kG>, kThreads, 0) != cudaSuccess || b < 1)
      b = 4;
    if (dev >= 0 && dev < 64) per_sm[dev].store(b, std::memory_order_relaxed);
  }
  const int64_t cap = static_cast<int64_t>(sm_count()) * b;
  if (blocks > cap) blocks = cap;
  score_kernel<L, kV, kG><<<static_cast<unsigned>(blocks), kThreads, 0, st>>>(x, xr, xp, HW, C, N, score);
}

// Motion-robust inter-frame score ([LIPAR] 2.B, short- and long-term
// differences): s = max(rel-L1 vs frame f-1, rel-L1 vs key frame max(f-L, 0)),
// frame 0 = +inf. Same lane layout as score_kernel; three rows per token (the
// two references were read moments before by other warps and come from L2).
template <int L, int kV>
__global__ void __launch_bounds__(256) score_motion_kernel(const uint16_t* __restrict__ x, int64_t HW, int64_t N,
                                                           int Lkey, float* __restrict__ score) {
  constexpr int kTokPerWarp = 32 / L;
  constexpr int C = kV * 8;
  const int lane = threadIdx.x & 31;
  const int sub = lane & (L - 1);
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t w0 = warp * kTokPerWarp; w0 < N; w0 += nwarps * kTokPerWarp) {
    const int64_t t = w0 + lane / L;
    const bool valid = t < N;
    const int64_t f = valid ? t / HW : 0;
    const bool first = f == 0;
    float n1 = 0.f, d1 = 0.f, n2 = 0.f, d2 = 0.f;
    if (valid && !first) {
      const int64_t fl = f - Lkey > 0 ? f - Lkey : 0;
      const uint16_t* cur = x + t * C;
      const uint16_t* r1 = x + (t - HW) * C;
      const uint16_t* r2 = x + (t - (f - fl) * HW) * C;
#pragma unroll
      for (int v = sub; v < kV; v += L) {
        const uint4 a = ld16(cur + v * 8), b = ld16(r1 + v * 8), c = ld16(r2 + v * 8);
        const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, bw[4] = {b.x, b.y, b.z, b.w}, cw[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float c0 = bf16lo(aw[i]), c1 = bf16hi(aw[i]);
          const float p0 = bf16lo(bw[i]), p1 = bf16hi(bw[i]);
          const float k0 = bf16lo(cw[i]), k1 = bf16hi(cw[i]);
          n1 += fabsf(c0 - p0) + fabsf(c1 - p1);
          d1 += fabsf(p0) + fabsf(p1);
          n2 += fabsf(c0 - k0) + fabsf(c1 - k1);
          d2 += fabsf(k0) + fabsf(k1);
        }
      }
    }
#pragma unroll
    for (int o = L / 2; o > 0; o >>= 1) {
      n1 += __shfl_xor_sync(0xffffffffu, n1, o);
      d1 += __shfl_xor_sync(0xffffffffu, d1, o);
      n2 += __shfl_xor_sync(0xffffffffu, n2, o);
      d2 += __shfl_xor_sync(0xffffffffu, d2, o);
    }
    if (valid && sub == 0) {
      auto ratio = [](float n, float d) { return d > 0.f ? n / d : (n > 0.f ? INFINITY : 0.f); };
      score[t] = first ? INFINITY : fmaxf(ratio(n1, d1), ratio(n2, d2));
    }
  }
}

}  // namespace
}  // namespace tps

extern "C" int lipar_score_motion(const tps_bf16* x, int64_t F, int64_t HW, int64_t C, int L, float* score,
                                  tps_stream stream) {
  TPS_TRACE("lipar_score_motion");
  using namespace tps;
  if (!x || !score) return fail(TPS_ERR_INVALID_ARG, "lipar_score_motion: x and score must be non-null");
  if (F < 1 || HW < 1 || F > (INT64_C(1) << 31) / HW) return fail(TPS_ERR_SHAPE, "lipar_score_motion: bad F/HW");
  if (C != 64 && C != 128) return fail(TPS_ERR_SHAPE, "lipar_score_motion: C=%lld must be 64 or 128", (long long)C);
  if (L < 1) return fail(TPS_ERR_INVALID_ARG, "lipar_score_motion: L=%d must be >= 1", L);
  if (!aligned16(x)) return fail(TPS_ERR_ALIGN, "lipar_score_motion: x must be 16-byte aligned");
  const int64_t N = F * HW;
  constexpr int kThreads = 256;
  const int64_t tok_per_block = (kThreads / 32) * 4;
  int64_t blocks = (N + tok_per_block - 1) / tok_per_block;
  const int64_t cap = static_cast<int64_t>(sm_count()) * 8;
  if (blocks > cap) blocks = cap;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (C == 128) score_motion_kernel<8, 16><<<static_cast<unsigned>(blocks), kThreads, 0, st>>>(x, HW, N, L, score);
  else score_motion_kernel<8, 8><<<static_cast<unsigned>(blocks), kThreads, 0, st>>>(x, HW, N, L, score);
  if (int e = launch_status("lipar_score_motion")) return e;
  return ok();
}

extern "C" int lipar_score(const tps_bf16* x, const tps_bf16* x_ref, const tps_bf16* x_prev_frame,
                           int64_t F, int64_t HW, int64_t C, float* score, tps_stream stream) {
  TPS_TRACE("lipar_score");
  using namespace tps;
  if (!x || !score) return fail(TPS_ERR_INVALID_ARG, "lipar_score: x and score must be non-null");
  if (F < 1 || HW < 1) return fail(TPS_ERR_SHAPE, "lipar_score: F=%lld HW=%lld must be >= 1",
                                   (long long)F, (long long)HW);
  if (C < 8 || C > 4096 || C % 8) return fail(TPS_ERR_SHAPE, "lipar_score: C=%lld must be a multiple of 8 in [8, 4096]", (long long)C);
  if (F > (INT64_C(1) << 31) / HW) return fail(TPS_ERR_SHAPE, "lipar_score: F*HW must be < 2^31");
  if (!aligned16(x) || (x_ref && !aligned16(x_ref)) || (x_prev_frame && !aligned16(x_prev_frame)))
    return fail(TPS_ERR_ALIGN, "lipar_score: bf16 inputs must be 16-byte aligned");
  if (x_ref && x_prev_frame) return fail(TPS_ERR_INVALID_ARG, "lipar_score: x_prev_frame is for inter-frame mode only");
  const int64_t N = F * HW;
  const int V = static_cast<int>(C / 8);
  const uint16_t* a = x;
  const uint16_t* r = x_ref;
  const uint16_t* p = x_prev_frame;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int c = static_cast<int>(C);
  if (c == 128) launch_score<8, 16, 2>(a, r, p, HW, c, N, score, st);
  else if (c == 64) launch_score<8, 8, 2>(a, r, p, HW, c, N, score, st);
  else if (c == 256) launch_score<8, 32, 2>(a, r, p, HW, c, N, score, st);
  else if (V >= 8) launch_score<8, 0, 2>(a, r, p, HW, c, N, score, st);
  else if (V >= 4) launch_score<4, 0, 2>(a, r, p, HW, c, N, score, st);
  else if (V >= 2) launch_score<2, 0, 2>(a, r, p, HW, c, N, score, st);
  else launch_score<1, 0, 2>(a, r, p, HW, c, N, score, st);
  if (int e = launch_status("lipar_score")) return e;
  return ok();
}
