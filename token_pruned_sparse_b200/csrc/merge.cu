// attn_lse_merge: exact merge of two attention results over disjoint key sets.
//
// [LIPAR] "Training-free Latent Inter-Frame Pruning with Attention Recovery",
// 2.C (Spanish summary): the attention of removed tokens is recovered with a
// log-sum-exp based combination. With w_i = exp(lse_i):
//     o = (w1 o1 + w2 o2) / (w1 + w2),   lse = log(w1 + w2),
// computed against m = max(lse1, lse2) so no exponential overflows. The same
// merge assembles split-key attention (two pruned_attn calls over two key
// ranges). HBM-bound elementwise pass: one thread per 16-byte vector of o.
#include <cmath>

#include "trace.cuh"
#include "tps_internal.cuh"

namespace tps {
namespace {

template <int kVpd>   // 16-byte vectors per head row (d / 8)
__global__ void __launch_bounds__(256) lse_merge_kernel(const uint4* __restrict__ o1, const float* __restrict__ l1,
                                                        const uint4* __restrict__ o2, const float* __restrict__ l2,
                                                        uint4* o, float* __restrict__ l, const int32_t* count,
                                                        int64_t cap, int H) {
  const int64_t rows = active_count(count, cap);
  const int64_t total = rows * H * kVpd;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t f = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; f < total; f += stride) {
    const int64_t rh = f / kVpd;
    const float a1 = l1[rh], a2 = l2[rh];
    const float m = fmaxf(a1, a2);
    uint4 out = make_uint4(0u, 0u, 0u, 0u);
    float lse = -INFINITY;
    if (m != -INFINITY) {
      const float w1 = expf(a1 - m), w2 = expf(a2 - m);   // exp(-inf) = 0 for an empty part
      const float sum = w1 + w2;
      const float c1 = w1 / sum, c2 = w2 / sum;
      const uint4 x = o1[f], y = o2[f];
      const uint32_t xw[4] = {x.x, x.y, x.z, x.w};
      const uint32_t yw[4] = {y.x, y.y, y.z, y.w};
      uint32_t r[4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
        r[i] = pack_bf16x2(fmaf(c1, bf16lo(xw[i]), c2 * bf16lo(yw[i])), fmaf(c1, bf16hi(xw[i]), c2 * bf16hi(yw[i])));
      out = make_uint4(r[0], r[1], r[2], r[3]);
      lse = m + logf(sum);
    }
    o[f] = out;
    if (f % kVpd == 0 && l) l[rh] = lse;
  }
}

// S-way merge of the fp32 partials written by split-key attention:
// o = sum_s w_s o_s / sum_s w_s, w_s = exp(lse_s - max_s lse_s).
template <int kVpd>
__global__ void __launch_bounds__(256) merge_parts_kernel(const float4* __restrict__ op,
                                                          const float* __restrict__ lp, int S, int64_t cap, int H,
                                                          const int32_t* count, uint4* __restrict__ o,
                                                          float* __restrict__ l) {
  const int64_t rows = active_count(count, cap);
  const int64_t total = rows * H * kVpd;
  const int64_t plane = cap * H;                       // (row, head) pairs per split
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t f = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; f < total; f += stride) {
    const int64_t rh = f / kVpd;
    float m = -INFINITY;
    for (int s = 0; s < S; ++s) m = fmaxf(m, lp[s * plane + rh]);
    uint4 out = make_uint4(0u, 0u, 0u, 0u);
    float lse = -INFINITY;
    if (m != -INFINITY) {
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      float sum = 0.f;
      for (int s = 0; s < S; ++s) {
        const float w = expf(lp[s * plane + rh] - m);
        const float4 a = op[(s * plane * kVpd + f) * 2], b = op[(s * plane * kVpd + f) * 2 + 1];
        acc[0] = fmaf(w, a.x, acc[0]);
        acc[1] = fmaf(w, a.y, acc[1]);
        acc[2] = fmaf(w, a.z, acc[2]);
        acc[3] = fmaf(w, a.w, acc[3]);
        acc[4] = fmaf(w, b.x, acc[4]);
        acc[5] = fmaf(w, b.y, acc[5]);
        acc[6] = fmaf(w, b.z, acc[6]);
        acc[7] = fmaf(w, b.w, acc[7]);
        sum += w;
      }
      const float inv = 1.f / sum;
      out = make_uint4(pack_bf16x2(acc[0] * inv, acc[1] * inv), pack_bf16x2(acc[2] * inv, acc[3] * inv),
                       pack_bf16x2(acc[4] * inv, acc[5] * inv), pack_bf16x2(acc[6] * inv, acc[7] * inv));
      lse = m + logf(sum);
    }
    o[f] = out;
    if (l && f % kVpd == 0) l[rh] = lse;
  }
}

}  // namespace

int merge_split_parts(const float* o_part, const float* lse_part, int nsplit, const int32_t* count, int64_t cap,
                      int H, int d, uint16_t* o, float* lse, cudaStream_t st) {
  const int64_t vecs = cap * H * (d / 8);
  int64_t grid = (vecs + 255) / 256;
  const int64_t maxg = static_cast<int64_t>(sm_count()) * 16;
  if (grid > maxg) grid = maxg;
  if (grid < 1) return TPS_OK;
  const auto* op = reinterpret_cast<const float4*>(o_part);
  auto* oo = reinterpret_cast<uint4*>(o);
  if (d == 128) merge_parts_kernel<16><<<static_cast<unsigned>(grid), 256, 0, st>>>(op, lse_part, nsplit, cap, H, count, oo, lse);
  else merge_parts_kernel<8><<<static_cast<unsigned>(grid), 256, 0, st>>>(op, lse_part, nsplit, cap, H, count, oo, lse);
  return launch_status("pruned_attn_ws: merge");
}

}  // namespace tps

extern "C" int attn_lse_merge(const tps_bf16* o1, const float* lse1, const tps_bf16* o2, const float* lse2,
                              const int32_t* count, int64_t cap, int H, int d, tps_bf16* o, float* lse,
                              tps_stream stream) {
  TPS_TRACE("attn_lse_merge");
  using namespace tps;
  if (!o1 || !lse1 || !o2 || !lse2 || !count || !o) return fail(TPS_ERR_INVALID_ARG, "attn_lse_merge: null pointer");
  if (d != 64 && d != 128) return fail(TPS_ERR_INVALID_ARG, "attn_lse_merge: d=%d must be 64 or 128", d);
  if (H < 1 || cap < 0 || cap >= (INT64_C(1) << 31)) return fail(TPS_ERR_SHAPE, "attn_lse_merge: bad H or cap");
  if (lse && (lse == lse1 || lse == lse2)) return fail(TPS_ERR_INVALID_ARG, "attn_lse_merge: lse must not alias lse1/lse2");
  if (!aligned16(o1) || !aligned16(o2) || !aligned16(o)) return fail(TPS_ERR_ALIGN, "attn_lse_merge: o arrays must be 16-byte aligned");
  if (cap == 0) return ok();
  const int64_t vecs = cap * H * (d / 8);
  int64_t grid = (vecs + 255) / 256;
  const int64_t maxg = static_cast<int64_t>(sm_count()) * 16;
  if (grid > maxg) grid = maxg;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const auto* a = reinterpret_cast<const uint4*>(o1);
  const auto* b = reinterpret_cast<const uint4*>(o2);
  auto* c = reinterpret_cast<uint4*>(o);
  if (d == 128) lse_merge_kernel<16><<<static_cast<unsigned>(grid), 256, 0, st>>>(a, lse1, b, lse2, c, lse, count, cap, H);
  else lse_merge_kernel<8><<<static_cast<unsigned>(grid), 256, 0, st>>>(a, lse1, b, lse2, c, lse, count, cap, H);
  if (int e = launch_status("attn_lse_merge")) return e;
  return ok();
}
