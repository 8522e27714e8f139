// Shared host-side validation and device helpers for the two attention kernels.
#pragma once

#include "tps_internal.cuh"

namespace tps {

struct AttnArgs {
  const uint16_t* q;
  const uint16_t* k;
  const uint16_t* v;
  const int32_t* idx;
  const int32_t* count;
  int64_t cap;
  int64_t N;
  int H;
  int d;
  float scale;
  const uint8_t* bm;
  int nb;          // key blocks of 128 (mask side), 0 when dense
  uint16_t* o;
  float* lse;
};

// Validates the pruned_attn contract; fills `a`. Returns TPS_OK or an error.
inline int attn_validate(const char* who, const tps_bf16* q_act, const tps_bf16* k, const tps_bf16* v,
                         const int32_t* idx, const int32_t* count, int64_t cap, int64_t N, int H, int d,
                         float scale, const uint8_t* blockmask, int block, tps_bf16* o_act, float* lse,
                         AttnArgs* a) {
  if (!q_act || !k || !v || !idx || !count || !o_act) return fail(TPS_ERR_INVALID_ARG, "%s: null pointer", who);
  if (d != 64 && d != 128) return fail(TPS_ERR_INVALID_ARG, "%s: d=%d must be 64 or 128", who, d);
  if (H < 1 || H > 256) return fail(TPS_ERR_SHAPE, "%s: H=%d must be in [1, 256]", who, H);
  if (N < 1 || N >= (INT64_C(1) << 31) || cap < 0 || cap >= (INT64_C(1) << 31))
    return fail(TPS_ERR_SHAPE, "%s: need 1 <= N < 2^31 and 0 <= cap < 2^31", who);
  if (!(scale > 0.f) || scale == INFINITY) return fail(TPS_ERR_INVALID_ARG, "%s: scale must be finite and > 0", who);
  int nb = 0;
  if (blockmask) {
    if (block != 128) return fail(TPS_ERR_INVALID_ARG, "%s: block=%d, only 128 is supported", who, block);
    const int64_t nbl = (N + 127) / 128;
    if (nbl > 4096) return fail(TPS_ERR_SHAPE, "%s: masked mode supports N <= 4096*128", who);
    nb = static_cast<int>(nbl);
  }
  if (!aligned16(q_act) || !aligned16(k) || !aligned16(v) || !aligned16(o_act))
    return fail(TPS_ERR_ALIGN, "%s: q/k/v/o must be 16-byte aligned", who);
  a->q = q_act;
  a->k = k;
  a->v = v;
  a->idx = idx;
  a->count = count;
  a->cap = cap;
  a->N = N;
  a->H = H;
  a->d = d;
  a->scale = scale;
  a->bm = blockmask;
  a->nb = nb;
  a->o = o_act;
  a->lse = lse;
  return TPS_OK;
}

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Two fp32 values in one 64-bit register, for the packed f32x2 instructions.
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
// (a.lo * b.lo + c.lo, a.hi * b.hi + c.hi) in one packed instruction
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

// P = 2^(S * scale_log2 - base) for one row of a kN-column S tile (fp32 bits in sr), as bf16
// pairs into pk; returns the fp32 row sum. The exponentials run on the MUFU unit (ex2.approx).
template <int kN>
__device__ __forceinline__ float exp_row(const uint32_t (&sr)[kN], uint64_t sl2x2, float base,
                                         uint32_t (&pk)[kN / 2]) {
  const uint64_t nbase = f2_pack(-base, -base);
  uint64_t acc0 = f2_pack(0.f, 0.f), acc1 = acc0;
#pragma unroll
  for (int c = 0; c < kN; c += 4) {
    const uint64_t a01 = ffma2(f2_pack(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1])), sl2x2, nbase);
    const uint64_t a23 = ffma2(f2_pack(__uint_as_float(sr[c + 2]), __uint_as_float(sr[c + 3])), sl2x2, nbase);
    float a0, a1, a2, a3;
    f2_unpack(a01, a0, a1);
    f2_unpack(a23, a2, a3);
    const float p0 = fast_exp2(a0), p1 = fast_exp2(a1), p2 = fast_exp2(a2), p3 = fast_exp2(a3);
    acc0 = fadd2(acc0, f2_pack(p0, p1));
    acc1 = fadd2(acc1, f2_pack(p2, p3));
    pk[c >> 1] = pack_bf16x2(p0, p1);
    pk[(c >> 1) + 1] = pack_bf16x2(p2, p3);
  }
  float s0, s1, s2, s3;
  f2_unpack(acc0, s0, s1);
  f2_unpack(acc1, s2, s3);
  return (s0 + s1) + (s2 + s3);
}

constexpr float kLog2e = 1.4426950408889634074f;
constexpr float kLn2 = 0.69314718055994530942f;

}  // namespace tps
