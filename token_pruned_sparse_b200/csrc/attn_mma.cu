// pruned_attn_mma: the legacy warp-level (mma.sync m16n8k16) tensor-core path
// of the pruned attention, kept as the baseline for the tcgen05 kernel.
//
// [HSA] 2.2 (3)-(4): active queries attend the full cached K/V, cost
// O(|A_i| * N). Optional key-block sparsity in the style of [SVOO] part 2 /
// [TR] (skipped key tiles): the mask row is the query's original 128-token
// block.
//
// Flash-style online softmax: a CTA owns 64 compacted active queries of one
// head (16 per warp) and streams 64-key K/V tiles through shared memory with
// cp.async double buffering. In masked mode the CTA first builds the list of
// key blocks that any of its query blocks keeps and loads only those tiles.
#include "trace.cuh"
#include "attn_common.cuh"

namespace tps {
namespace {

constexpr int kBM = 64;   // queries per CTA
constexpr int kBN = 64;   // keys per tile
constexpr int kThreads = 128;

template <int D>
struct Smem {
  static constexpr int kQ = kBM * D;       // bf16 elements
  static constexpr int kKV = kBN * D;
  static constexpr size_t kBytes = (kQ + 4 * kKV) * 2;
};

// 16-byte chunk c of row r lives at chunk (c ^ (r & 7)): conflict-free ldmatrix.
template <int D>
__device__ __forceinline__ uint32_t swz(int r, int c) {
  return static_cast<uint32_t>(r * D + ((c ^ (r & 7)) << 3));
}

__device__ __forceinline__ void cp_async16(uint32_t saddr, const void* g, bool pred) {
  const int n = pred ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(saddr), "l"(g), "r"(n));
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;"); }
template <int N>
__device__ __forceinline__ void cp_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N)); }

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void mma16816(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

template <int D>
__global__ void __launch_bounds__(kThreads) attn_mma_kernel(AttnArgs p, float scale_log2) {
  extern __shared__ __align__(128) uint16_t smem[];
  uint16_t* sQ = smem;
  uint16_t* sK = sQ + Smem<D>::kQ;            // [2][kBN][D]
  uint16_t* sV = sK + 2 * Smem<D>::kKV;       // [2][kBN][D]
  uint16_t* sList = sV + 2 * Smem<D>::kKV;    // masked mode: kept 64-key tiles
  __shared__ int s_ntiles;
  __shared__ unsigned int s_wcnt[kThreads / 32];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int h = blockIdx.y;
  const int64_t rows = active_count(p.count, p.cap);
  const int64_t row0 = static_cast<int64_t>(blockIdx.x) * kBM;
  if (row0 >= rows) return;
  const int64_t H = p.H;
  const int64_t N = p.N;
  const int total_tiles = static_cast<int>((N + kBN - 1) / kBN);

  // ---- key-tile list (masked mode) -------------------------------------------------
  if (p.bm) {
    const int64_t rlast = (row0 + kBM - 1 < rows ? row0 + kBM - 1 : rows - 1);
    int qb0 = p.idx[row0] / 128, qb1 = p.idx[rlast] / 128;
    qb0 = qb0 < 0 ? 0 : (qb0 >= p.nb ? p.nb - 1 : qb0);
    qb1 = qb1 < qb0 ? qb0 : (qb1 >= p.nb ? p.nb - 1 : qb1);
    int base = 0;
    for (int kb0 = 0; kb0 < p.nb; kb0 += kThreads) {
      const int kb = kb0 + tid;
      bool keep = false;
      if (kb < p.nb)
        for (int qb = qb0; qb <= qb1 && !keep; ++qb) keep = p.bm[static_cast<int64_t>(qb) * p.nb + kb] != 0;
      const unsigned int m = __ballot_sync(0xffffffffu, keep);
      if (lane == 0) s_wcnt[warp] = __popc(m);
      __syncthreads();
      int off = base;
      for (int i = 0; i < warp; ++i) off += s_wcnt[i];
      int tot = 0;
      for (int i = 0; i < kThreads / 32; ++i) tot += s_wcnt[i];
      if (keep) {
        const int pos = off + __popc(m & ((1u << lane) - 1u));
        sList[2 * pos] = static_cast<uint16_t>(2 * kb);
        sList[2 * pos + 1] = static_cast<uint16_t>(2 * kb + 1);
      }
      base += tot;
      __syncthreads();
    }
    if (tid == 0) {
      int nt = 2 * base;
      // the second half of the last key block may lie beyond N
      if (nt > 0 && sList[nt - 1] >= total_tiles) --nt;
      s_ntiles = nt;
    }
    __syncthreads();
  } else if (tid == 0) {
    s_ntiles = total_tiles;
  }
  __syncthreads();
  const int ntiles = s_ntiles;

  // ---- Q tile -> shared -> registers ---------------------------------------------------
  constexpr int kChunks = D / 8;
  const uint32_t sQa = static_cast<uint32_t>(__cvta_generic_to_shared(sQ));
  const uint32_t sKa = static_cast<uint32_t>(__cvta_generic_to_shared(sK));
  const uint32_t sVa = static_cast<uint32_t>(__cvta_generic_to_shared(sV));
  for (int i = tid; i < kBM * kChunks; i += kThreads) {
    const int r = i / kChunks, c = i % kChunks;
    const int64_t row = row0 + r;
    const bool ok = row < rows;
    const uint16_t* g = p.q + ((ok ? row : 0) * H + h) * D + c * 8;
    cp_async16(sQa + swz<D>(r, c) * 2, g, ok);
  }
  cp_commit();

  auto tile_key0 = [&](int t) -> int64_t {
    return static_cast<int64_t>(p.bm ? sList[t] : t) * kBN;
  };
  auto load_kv = [&](int t, int stage) {
    const int64_t n0 = tile_key0(t);
    for (int i = tid; i < kBN * kChunks; i += kThreads) {
      const int r = i / kChunks, c = i % kChunks;
      const int64_t n = n0 + r;
      const bool ok = n < N;
      const int64_t off = ((ok ? n : 0) * H + h) * D + c * 8;
      const uint32_t so = (stage * Smem<D>::kKV + swz<D>(r, c)) * 2;
      cp_async16(sKa + so, p.k + off, ok);
      cp_async16(sVa + so, p.v + off, ok);
    }
  };
  if (ntiles > 0) load_kv(0, 0);
  cp_commit();

  // per-thread rows g and g+8 of this warp's 16
  const int g = lane >> 2, tig = lane & 3;
  int qblk[2] = {0, 0};
  if (p.bm) {
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      int64_t row = row0 + warp * 16 + g + i * 8;
      row = row < rows ? row : rows - 1;
      int qb = p.idx[row] / 128;
      qblk[i] = qb < 0 ? 0 : (qb >= p.nb ? p.nb - 1 : qb);
    }
  }

  cp_wait<1>();
  __syncthreads();
  uint32_t qf[D / 16][4];
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const int m = lane >> 3;
    const int r = warp * 16 + (m & 1) * 8 + (lane & 7);
    const int c = kk * 2 + (m >> 1);
    ldsm_x4(sQa + swz<D>(r, c) * 2, qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3]);
  }

  float acc[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
  float mrow[2] = {-INFINITY, -INFINITY};
  float lrow[2] = {0.f, 0.f};

  for (int t = 0; t < ntiles; ++t) {
    const int stage = t & 1;
    if (t + 1 < ntiles) load_kv(t + 1, stage ^ 1);
    cp_commit();
    cp_wait<1>();
    __syncthreads();

    const int64_t n0 = tile_key0(t);
    const uint32_t kbase = sKa + stage * Smem<D>::kKV * 2;
    const uint32_t vbase = sVa + stage * Smem<D>::kKV * 2;
    float s[kBN / 8][4];
#pragma unroll
    for (int i = 0; i < kBN / 8; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
      for (int pp = 0; pp < kBN / 16; ++pp) {
        const int m = lane >> 3;
        const int r = pp * 16 + (m >> 1) * 8 + (lane & 7);
        const int c = kk * 2 + (m & 1);
        uint32_t b0, b1, b2, b3;
        ldsm_x4(kbase + swz<D>(r, c) * 2, b0, b1, b2, b3);
        mma16816(s[2 * pp], qf[kk], b0, b1);
        mma16816(s[2 * pp + 1], qf[kk], b2, b3);
      }
    }
    // scale, mask, online softmax (log2 domain)
    bool row_ok[2] = {true, true};
    if (p.bm) {
      const int kb = static_cast<int>(n0 / 128);
#pragma unroll
      for (int i = 0; i < 2; ++i) row_ok[i] = p.bm[static_cast<int64_t>(qblk[i]) * p.nb + kb] != 0;
    }
    float tmax[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int nt = 0; nt < kBN / 8; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int i = e >> 1;
        const int64_t n = n0 + nt * 8 + tig * 2 + (e & 1);
        float x = s[nt][e] * scale_log2;
        if (n >= N || !row_ok[i]) x = -INFINITY;
        s[nt][e] = x;
        tmax[i] = fmaxf(tmax[i], x);
      }
    }
    float alpha[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      tmax[i] = fmaxf(tmax[i], __shfl_xor_sync(0xffffffffu, tmax[i], 1));
      tmax[i] = fmaxf(tmax[i], __shfl_xor_sync(0xffffffffu, tmax[i], 2));
      const float mnew = fmaxf(mrow[i], tmax[i]);
      alpha[i] = mnew == -INFINITY ? 1.f : fast_exp2(mrow[i] - mnew);
      mrow[i] = mnew;
    }
    float psum[2] = {0.f, 0.f};
    uint32_t pf[kBN / 16][4];
#pragma unroll
    for (int nt = 0; nt < kBN / 8; ++nt) {
      float pv[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int i = e >> 1;
        const float base = mrow[i] == -INFINITY ? 0.f : mrow[i];
        pv[e] = fast_exp2(s[nt][e] - base);
        psum[i] += pv[e];
      }
      pf[nt >> 1][(nt & 1) * 2 + 0] = pack_bf16x2(pv[0], pv[1]);
      pf[nt >> 1][(nt & 1) * 2 + 1] = pack_bf16x2(pv[2], pv[3]);
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) lrow[i] = lrow[i] * alpha[i] + psum[i];
#pragma unroll
    for (int dt = 0; dt < D / 8; ++dt) {
      acc[dt][0] *= alpha[0];
      acc[dt][1] *= alpha[0];
      acc[dt][2] *= alpha[1];
      acc[dt][3] *= alpha[1];
    }
    // O += P V
#pragma unroll
    for (int kk = 0; kk < kBN / 16; ++kk) {
      const uint32_t a[4] = {pf[kk][0], pf[kk][1], pf[kk][2], pf[kk][3]};
#pragma unroll
      for (int dp = 0; dp < D / 16; ++dp) {
        const int m = lane >> 3;
        const int r = kk * 16 + (m & 1) * 8 + (lane & 7);
        const int c = dp * 2 + (m >> 1);
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(vbase + swz<D>(r, c) * 2, b0, b1, b2, b3);
        mma16816(acc[2 * dp], a, b0, b1);
        mma16816(acc[2 * dp + 1], a, b2, b3);
      }
    }
    __syncthreads();
  }

  // ---- epilogue ---------------------------------------------------------------------------
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    lrow[i] += __shfl_xor_sync(0xffffffffu, lrow[i], 1);
    lrow[i] += __shfl_xor_sync(0xffffffffu, lrow[i], 2);
  }
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int64_t row = row0 + warp * 16 + g + i * 8;
    if (row >= rows) continue;
    const float inv = lrow[i] > 0.f ? 1.f / lrow[i] : 0.f;
    uint32_t* orow = reinterpret_cast<uint32_t*>(p.o + (row * H + h) * D);
#pragma unroll
    for (int dt = 0; dt < D / 8; ++dt)
      orow[(dt * 8 + tig * 2) / 2] = pack_bf16x2(acc[dt][2 * i] * inv, acc[dt][2 * i + 1] * inv);
    if (p.lse && tig == 0)
      p.lse[row * H + h] = lrow[i] > 0.f ? (mrow[i] + __log2f(lrow[i])) * kLn2 : -INFINITY;
  }
}

template <int D>
int launch(const AttnArgs& a, cudaStream_t st) {
  if (a.cap == 0) return TPS_OK;
  size_t smem = Smem<D>::kBytes;
  if (a.bm) smem += static_cast<size_t>(a.nb) * 2 * sizeof(uint16_t);
  static std::atomic<bool> attr_set[64];   // the attribute is per device
  int dev = 0;
  cudaGetDevice(&dev);
  const bool cached = dev >= 0 && dev < 64 && attr_set[dev].load(std::memory_order_acquire);
  if (!cached) {
    cudaError_t e = cudaFuncSetAttribute(attn_mma_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(Smem<D>::kBytes + 4096 * 2 * sizeof(uint16_t)));
    if (e != cudaSuccess) return cuda_status(e, "pruned_attn_mma: smem attribute");
    if (dev >= 0 && dev < 64) attr_set[dev].store(true, std::memory_order_release);
  }
  dim3 grid(static_cast<unsigned int>((a.cap + kBM - 1) / kBM), static_cast<unsigned int>(a.H));
  attn_mma_kernel<D><<<grid, kThreads, smem, st>>>(a, a.scale * kLog2e);
  return launch_status("pruned_attn_mma");
}

}  // namespace
}  // namespace tps

extern "C" int pruned_attn_mma(const tps_bf16* q_act, const tps_bf16* k, const tps_bf16* v,
                               const int32_t* idx, const int32_t* count, int64_t cap, int64_t N, int H,
                               int d, float scale, const uint8_t* blockmask, int block, tps_bf16* o_act,
                               float* lse, tps_stream stream) {
  TPS_TRACE("pruned_attn_mma");
  using namespace tps;
  AttnArgs a;
  if (int e = attn_validate("pruned_attn_mma", q_act, k, v, idx, count, cap, N, H, d, scale, blockmask,
                            block, o_act, lse, &a))
    return e;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int e = d == 64 ? launch<64>(a, st) : launch<128>(a, st);
  return e ? e : ok();
}
