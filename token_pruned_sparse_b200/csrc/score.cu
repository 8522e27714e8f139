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

#include "tps_internal.cuh"

namespace tps {
namespace {

template <int L>
__global__ void __launch_bounds__(256) score_kernel(const uint16_t* __restrict__ x,
                                                    const uint16_t* __restrict__ xref,
                                                    const uint16_t* __restrict__ xprev,
                                                    int64_t HW, int C, int64_t N,
                                                    float* __restrict__ score) {
  constexpr int kTokPerWarp = 32 / L;
  const int lane = threadIdx.x & 31;
  const int sub = lane & (L - 1);
  const int V = C >> 3;  // 16-byte vectors per row
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t w0 = warp * kTokPerWarp; w0 < N; w0 += nwarps * kTokPerWarp) {
    const int64_t t = w0 + lane / L;
    const bool valid = t < N;
    const uint16_t* ref = nullptr;
    if (valid) {
      if (xref) ref = xref + t * C;
      else if (t >= HW) ref = x + (t - HW) * C;
      else if (xprev) ref = xprev + t * C;
    }
    float num = 0.f, den = 0.f;
    if (ref) {
      const uint16_t* cur = x + t * C;
#pragma unroll 4
      for (int v = sub; v < V; v += L) {
        const uint4 a = ld16(cur + v * 8);
        const uint4 b = ld16(ref + v * 8);
        const uint32_t aw[4] = {a.x, a.y, a.z, a.w};
        const uint32_t bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float c0 = bf16lo(aw[i]), c1 = bf16hi(aw[i]);
          const float r0 = bf16lo(bw[i]), r1 = bf16hi(bw[i]);
          num += fabsf(c0 - r0) + fabsf(c1 - r1);
          den += fabsf(r0) + fabsf(r1);
        }
      }
    }
#pragma unroll
    for (int o = L / 2; o > 0; o >>= 1) {
      num += __shfl_xor_sync(0xffffffffu, num, o);
      den += __shfl_xor_sync(0xffffffffu, den, o);
    }
    if (valid && sub == 0) {
      float s;
      if (!ref) s = INFINITY;                       // frame 0 without a predecessor
      else if (den > 0.f) s = num / den;
      else s = num > 0.f ? INFINITY : 0.f;
      score[t] = s;
    }
  }
}

template <int L>
void launch_score(const uint16_t* x, const uint16_t* xr, const uint16_t* xp, int64_t HW, int C,
                  int64_t N, float* score, cudaStream_t st) {
  constexpr int kThreads = 256;
  const int64_t tok_per_block = (kThreads / 32) * (32 / L);
  int64_t blocks = (N + tok_per_block - 1) / tok_per_block;
  const int64_t cap = static_cast<int64_t>(sm_count()) * 16;
  if (blocks > cap) blocks = cap;
  score_kernel<L><<<static_cast<unsigned>(blocks), kThreads, 0, st>>>(x, xr, xp, HW, C, N, score);
}

}  // namespace
}  // namespace tps

extern "C" int lipar_score(const tps_bf16* x, const tps_bf16* x_ref, const tps_bf16* x_prev_frame,
                           int64_t F, int64_t HW, int64_t C, float* score, tps_stream stream) {
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
  if (V >= 8) launch_score<8>(a, r, p, HW, c, N, score, st);
  else if (V >= 4) launch_score<4>(a, r, p, HW, c, N, score, st);
  else if (V >= 2) launch_score<2>(a, r, p, HW, c, N, score, st);
  else launch_score<1>(a, r, p, HW, c, N, score, st);
  if (int e = launch_status("lipar_score")) return e;
  return ok();
}
