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

constexpr float kLog2e = 1.4426950408889634074f;
constexpr float kLn2 = 0.69314718055994530942f;

}  // namespace tps
