// pruned_attn: active queries attend all N cached keys, on the Blackwell
// tensor cores (tcgen05 + TMEM + TMA).
//
// [HSA] "Asignacion de Pasos Heterogenea", 2.2 (3)-(4): the active tokens'
// queries attend the full cached K/V (fresh rows for active tokens, stale but
// valid rows for skipped ones), so the attention costs O(|A_i| * N).
// Key-block sparsity ([SVOO] part 2, co-clustering -> block-sparse attention;
// [TR] skipping of reusable work): with a mask, a query attends only the
// 128-key blocks its ORIGINAL 128-token block keeps; whole key tiles that no
// query of a CTA needs are never loaded.
//
// Kernel layout (one CTA = 128 compacted active queries x one head):
//   warps 0-3  softmax: thread r owns query row r (= TMEM lane r). Reads S from
//              TMEM, applies scale / masks / online softmax in the log2 domain,
//              rescales O in TMEM when the running max grows, writes P (bf16) to
//              shared memory, and finally normalises O and stores it.
//   warp 4     TMA producer: Q once, then K and V tiles (128 keys each) into a
//              two-stage ring, 128-byte swizzled.
//   warp 5     MMA issuer and TMEM owner: S_j = Q K_j^T into one of two TMEM S
//              buffers, O += P_j V_j into the TMEM O accumulator; completion is
//              signalled with tcgen05.commit on mbarriers.
// S_{j+1} is issued as soon as its buffer is free, so the tensor cores compute
// S_{j+1} and P_j V_j while the softmax warps work on tile j+1.
// Every mbarrier wait is bounded: on expiry the CTA sets an abort flag and the
// device status word (TPS_ERR_TIMEOUT via tps_check), drains what it issued,
// frees TMEM and returns.
#include <mutex>

#include "attn_common.cuh"
#include "tc_ptx.cuh"

namespace tps {
namespace {

using namespace tc;

constexpr int kBM = 128;        // queries per CTA (MMA M)
constexpr int kBN = 128;        // keys per tile (MMA N of S, K of PV)
constexpr int kStages = 2;      // K/V ring depth
constexpr int kThreads = 192;   // 4 softmax warps + TMA warp + MMA warp
constexpr int kTmemCols = 512;  // S0 | S1 | O
constexpr int kSubBytes = kBN * 128;   // one [128 rows x 64 bf16] swizzled sub-tile

template <int D>
struct Layout {
  static constexpr int kSub = D / 64;                    // 64-wide sub-tiles per row of Q/K/V
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + kSub * kSubBytes;       // [stage][sub]
  static constexpr int kV = kK + kStages * kSub * kSubBytes;
  static constexpr int kP = kV + kStages * kSub * kSubBytes;   // 2 sub-tiles (128 keys)
  static constexpr int kList = kP + 2 * kSubBytes;       // uint16 kept key blocks
  static constexpr int kListMax = 4096;
  static constexpr int kBar = kList + kListMax * 2;      // mbarriers (Bars)
  static constexpr int kBytes = kBar + 256;
  static constexpr int kAlloc = kBytes + 1024;           // slack for 1024-byte alignment
};

struct Bars {  // mbarrier offsets inside the barrier block (8 bytes each)
  static constexpr int q_full = 0;
  static constexpr int k_full = 1;            // + stage
  static constexpr int v_full = 1 + kStages;  // + stage
  static constexpr int kv_empty = 1 + 2 * kStages;
  static constexpr int s_full = 1 + 3 * kStages;   // + buffer (2)
  static constexpr int s_free = 3 + 3 * kStages;   // + buffer (2)
  static constexpr int p_full = 5 + 3 * kStages;
  static constexpr int pv_done = 6 + 3 * kStages;
  static constexpr int drain = 7 + 3 * kStages;    // last commit of the MMA thread
};

struct TcParams {
  AttnArgs a;
  float scale_log2;
  unsigned int* status;
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, TcParams prm) {
  using L = Layout<D>;
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint32_t s_tmem;
  __shared__ int s_ntiles;
  __shared__ volatile int s_abort;
  __shared__ unsigned int s_wcnt[kThreads / 32];

  const AttnArgs& p = prm.a;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.y;
  const int64_t rows = active_count(p.count, p.cap);
  const int64_t row0 = static_cast<int64_t>(blockIdx.x) * kBM;
  if (row0 >= rows) return;   // whole CTA exits before touching TMEM or barriers

  const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (sbase - smem_u32(smem_raw));
  uint16_t* sList = reinterpret_cast<uint16_t*>(gbase + L::kList);
  const uint32_t bar0 = sbase + L::kBar;
  auto bar = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };
  const int nkt = static_cast<int>((p.N + kBN - 1) / kBN);   // key tiles = key blocks

  // ---- setup: barriers, TMEM, key-tile list ---------------------------------------------
  if (tid == 0) {
    s_abort = 0;
    mbar_init(bar(Bars::q_full), 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(Bars::k_full + s), 1);
      mbar_init(bar(Bars::v_full + s), 1);
      mbar_init(bar(Bars::kv_empty + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(Bars::s_full + b), 1);
      mbar_init(bar(Bars::s_free + b), kBM);
    }
    mbar_init(bar(Bars::p_full), kBM);
    mbar_init(bar(Bars::pv_done), 1);
    mbar_init(bar(Bars::drain), 1);
    fence_mbar_init();
  }
  if (warp == 5) tmem_alloc<kTmemCols>(smem_u32(&s_tmem));
  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  if (p.bm) {
    const int64_t rlast = row0 + kBM - 1 < rows ? row0 + kBM - 1 : rows - 1;
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
      int off = base, tot = 0;
      for (int i = 0; i < kThreads / 32; ++i) {
        off += i < warp ? s_wcnt[i] : 0;
        tot += s_wcnt[i];
      }
      if (keep) sList[off + __popc(m & ((1u << lane) - 1u))] = static_cast<uint16_t>(kb);
      base += tot;
      __syncthreads();
    }
    if (tid == 0) s_ntiles = base;
  } else if (tid == 0) {
    s_ntiles = nkt;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const int ntiles = s_ntiles;
  const uint32_t tmem = s_tmem;
  const uint32_t tS = tmem;            // S buffer b at column 128 * b
  const uint32_t tO = tmem + 256;      // O accumulator, D columns
  auto tile_kb = [&](int j) -> int { return p.bm ? static_cast<int>(sList[j]) : j; };

  if (warp == 4) {
    // ================================ TMA producer =====================================
    if (lane == 0) {
      int issued = 0;
      mbar_expect_tx(bar(Bars::q_full), L::kSub * kSubBytes);
      for (int s = 0; s < L::kSub; ++s)
        tma_load_3d(sbase + L::kQ + s * kSubBytes, &tmQ, 64 * s, h, static_cast<int>(row0), bar(Bars::q_full));
      for (int j = 0; j < ntiles; ++j) {
        const int st = j % kStages;
        if (j >= kStages && !mbar_wait(bar(Bars::kv_empty + st), ((j / kStages) - 1) & 1, &s_abort, prm.status))
          break;
        const int key0 = tile_kb(j) * kBN;
        mbar_expect_tx(bar(Bars::k_full + st), L::kSub * kSubBytes);
        for (int s = 0; s < L::kSub; ++s)
          tma_load_3d(sbase + L::kK + (st * L::kSub + s) * kSubBytes, &tmK, 64 * s, h, key0, bar(Bars::k_full + st));
        mbar_expect_tx(bar(Bars::v_full + st), L::kSub * kSubBytes);
        for (int s = 0; s < L::kSub; ++s)
          tma_load_3d(sbase + L::kV + (st * L::kSub + s) * kSubBytes, &tmV, 64 * s, h, key0, bar(Bars::v_full + st));
        issued = j + 1;
      }
      // drain: every load issued above must land before the CTA may exit
      drain_wait(bar(Bars::q_full), 0);
      for (int j = issued > kStages ? issued - kStages : 0; j < issued; ++j) {
        drain_wait(bar(Bars::k_full + j % kStages), (j / kStages) & 1);
        drain_wait(bar(Bars::v_full + j % kStages), (j / kStages) & 1);
      }
    }
  } else if (warp == 5) {
    // ================================ MMA issuer =======================================
    if (lane == 0) {
      constexpr uint32_t kIdescS = idesc_bf16(kBM, kBN, false, false);  // Q K^T: both K-major
      constexpr uint32_t kIdescO = idesc_bf16(kBM, D, false, true);     // P V: V is MN-major
      bool ok = mbar_wait(bar(Bars::q_full), 0, &s_abort, prm.status);
      tc_fence_after();
      auto issue_s = [&](int j) -> bool {
        const int st = j % kStages, b = j & 1;
        if (!mbar_wait(bar(Bars::k_full + st), (j / kStages) & 1, &s_abort, prm.status)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kSubBytes + (kk & 3) * 32;   // 16 bf16 along d
          const uint64_t da = sdesc_sw128(sbase + L::kQ + off, 16, 1024);
          const uint64_t db = sdesc_sw128(sbase + L::kK + st * L::kSub * kSubBytes + off, 16, 1024);
          mma_f16_ss(tS + 128 * b, da, db, kIdescS, kk > 0);
        }
        mma_commit(bar(Bars::s_full + b));
        return true;
      };
      if (ok && ntiles > 0) ok = issue_s(0);
      for (int j = 0; ok && j < ntiles; ++j) {
        if (j + 1 < ntiles) {
          if (j + 1 >= 2) {
            ok = mbar_wait(bar(Bars::s_free + ((j + 1) & 1)), (((j + 1) >> 1) - 1) & 1, &s_abort, prm.status);
            tc_fence_after();
          }
          if (ok) ok = issue_s(j + 1);
          if (!ok) break;
        }
        const int st = j % kStages;
        if (!mbar_wait(bar(Bars::p_full), j & 1, &s_abort, prm.status)) break;
        if (!mbar_wait(bar(Bars::v_full + st), (j / kStages) & 1, &s_abort, prm.status)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk) {
          // A = P [128 q x 128 keys], K-major (keys contiguous): 16 keys per step
          const uint64_t da = sdesc_sw128(sbase + L::kP + (kk >> 2) * kSubBytes + (kk & 3) * 32, 16, 1024);
          // B = V [128 keys x D], MN-major: 16 keys = 2 swizzle atoms of 8 rows;
          // LBO = next 64-wide d sub-tile, SBO = next 8 keys
          const uint64_t db = sdesc_sw128(sbase + L::kV + st * L::kSub * kSubBytes + kk * 16 * 128, kSubBytes, 1024);
          mma_f16_ss(tO, da, db, kIdescO, (j > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(bar(Bars::pv_done));
        mma_commit(bar(Bars::kv_empty + st));
      }
      mma_commit(bar(Bars::drain));   // fires once every MMA issued above has completed
    }
  } else {
    // ================================ softmax warps ====================================
    const int r = tid;                            // query row within the tile == TMEM lane
    const int64_t row = row0 + r;
    const bool valid = row < rows;
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    int qb = 0;
    if (p.bm) {
      qb = p.idx[valid ? row : rows - 1] / 128;
      qb = qb < 0 ? 0 : (qb >= p.nb ? p.nb - 1 : qb);
    }
    const float sl2 = prm.scale_log2;
    float m_run = -INFINITY, l_run = 0.f;
    uint8_t* sP = gbase + L::kP;
    bool ok = true;
    for (int j = 0; j < ntiles; ++j) {
      const int b = j & 1;
      // every wait result is made warp-uniform: tcgen05.ld/st are .sync.aligned
      if (!__all_sync(0xffffffffu, mbar_wait(bar(Bars::s_full + b), (j >> 1) & 1, &s_abort, prm.status))) {
        ok = false;
        break;
      }
      tc_fence_after();
      float s[kBN];
#pragma unroll
      for (int c = 0; c < kBN / 32; ++c) tmem_ld32(tS + 128 * b + 32 * c + lane_off, s + 32 * c);
      tc_fence_before();
      mbar_arrive(bar(Bars::s_free + b));

      const int kb = tile_kb(j);
      const int64_t key0 = static_cast<int64_t>(kb) * kBN;
      const bool row_ok = !p.bm || p.bm[static_cast<int64_t>(qb) * p.nb + kb] != 0;
      const int nvalid = row_ok ? static_cast<int>(p.N - key0 < kBN ? p.N - key0 : kBN) : 0;
      float tmax = -INFINITY;
#pragma unroll
      for (int c = 0; c < kBN; ++c) {
        const float x = c < nvalid ? s[c] * sl2 : -INFINITY;
        s[c] = x;
        tmax = fmaxf(tmax, x);
      }
      const float m_new = fmaxf(m_run, tmax);
      const float base = m_new == -INFINITY ? 0.f : m_new;
      const float alpha = m_run == -INFINITY ? (j == 0 ? 1.f : 0.f) : fast_exp2(m_run - m_new);
      float psum = 0.f;
      uint32_t pk[kBN / 2];
#pragma unroll
      for (int c = 0; c < kBN; c += 2) {
        const float p0 = fast_exp2(s[c] - base), p1 = fast_exp2(s[c + 1] - base);
        psum += p0 + p1;
        pk[c >> 1] = pack_bf16x2(p0, p1);
      }
      l_run = l_run * alpha + psum;
      m_run = m_new;

      if (j > 0) {
        // PV_{j-1} must be complete before O is rescaled and before P is overwritten
        if (!__all_sync(0xffffffffu, mbar_wait(bar(Bars::pv_done), (j - 1) & 1, &s_abort, prm.status))) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (__any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            float o[32];
            tmem_ld32(tO + 32 * c + lane_off, o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] *= alpha;
            tmem_st32(tO + 32 * c + lane_off, o);
          }
        }
      }
      // P row r -> two K-major swizzled sub-tiles (keys 0-63, 64-127)
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const int sub = c >> 3, cc = c & 7;
        uint4 v = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
        *reinterpret_cast<uint4*>(sP + sub * kSubBytes + r * 128 + ((cc ^ (r & 7)) << 4)) = v;
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar(Bars::p_full));
    }
    // ---- epilogue ------------------------------------------------------------------------
    if (ok && ntiles > 0) ok = mbar_wait(bar(Bars::pv_done), (ntiles - 1) & 1, &s_abort, prm.status);
    ok = __all_sync(0xffffffffu, ok);
    tc_fence_after();
    if (ok) {
      const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
      uint4* orow = reinterpret_cast<uint4*>(p.o + (row * p.H + h) * D);
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        float o[32];
        if (ntiles > 0) tmem_ld32(tO + 32 * c + lane_off, o);
        else
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = 0.f;
        if (valid) {
#pragma unroll
          for (int q = 0; q < 4; ++q)
            orow[4 * c + q] = make_uint4(pack_bf16x2(o[8 * q + 0] * inv, o[8 * q + 1] * inv),
                                         pack_bf16x2(o[8 * q + 2] * inv, o[8 * q + 3] * inv),
                                         pack_bf16x2(o[8 * q + 4] * inv, o[8 * q + 5] * inv),
                                         pack_bf16x2(o[8 * q + 6] * inv, o[8 * q + 7] * inv));
        }
      }
      if (valid && p.lse) p.lse[row * p.H + h] = l_run > 0.f ? (m_run + __log2f(l_run)) * kLn2 : -INFINITY;
    }
  }

  // ---- teardown ------------------------------------------------------------------------
  if (warp == 5 && lane == 0) drain_wait(bar(Bars::drain), 0);   // no MMA may still write TMEM
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 5) {
    __syncwarp();
    tmem_dealloc<kTmemCols>(tmem);
  }
}

// ---- host ------------------------------------------------------------------------------------
using EncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                 const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

int get_encoder(EncodeTiled* fn) {
  static EncodeTiled cached = nullptr;
  static std::once_flag once;
  static int err = TPS_OK;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q);
    if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !f)
      err = fail(TPS_ERR_CUDA, "pruned_attn: cuTensorMapEncodeTiled unavailable (%s)", cudaGetErrorString(e));
    else
      cached = reinterpret_cast<EncodeTiled>(f);
  });
  *fn = cached;
  return cached ? TPS_OK : (err ? err : fail(TPS_ERR_CUDA, "pruned_attn: no tensor-map encoder"));
}

// [rows, H, d] bf16, token-major -> 3-D map (d, H, rows), box (64, 1, 128), 128-byte swizzle.
int make_map(EncodeTiled enc, CUtensorMap* m, const void* base, int64_t rows, int H, int d) {
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(H) * d * 2};
  cuuint32_t box[3] = {64, 1, 128};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(TPS_ERR_CUDA, "pruned_attn: cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return TPS_OK;
}

template <int D>
int launch(const AttnArgs& a, cudaStream_t st) {
  if (a.cap == 0) return TPS_OK;
  EncodeTiled enc;
  if (int e = get_encoder(&enc)) return e;
  int err;
  unsigned int* status = device_status(&err);
  if (!status) return err;
  CUtensorMap mq, mk, mv;
  if (int e = make_map(enc, &mq, a.q, a.cap, a.H, a.d)) return e;
  if (int e = make_map(enc, &mk, a.k, a.N, a.H, a.d)) return e;
  if (int e = make_map(enc, &mv, a.v, a.N, a.H, a.d)) return e;
  constexpr int kSmem = Layout<D>::kAlloc;
  static bool attr_done[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_done[dev]) {
    cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    if (e != cudaSuccess) return cuda_status(e, "pruned_attn: smem attribute");
    attr_done[dev] = true;
  }
  TcParams prm{a, a.scale * kLog2e, status};
  dim3 grid(static_cast<unsigned int>((a.cap + kBM - 1) / kBM), static_cast<unsigned int>(a.H));
  attn_tc_kernel<D><<<grid, kThreads, kSmem, st>>>(mq, mk, mv, prm);
  return launch_status("pruned_attn");
}

}  // namespace
}  // namespace tps

extern "C" int pruned_attn(const tps_bf16* q_act, const tps_bf16* k, const tps_bf16* v, const int32_t* idx,
                           const int32_t* count, int64_t cap, int64_t N, int H, int d, float scale,
                           const uint8_t* blockmask, int block, tps_bf16* o_act, float* lse, tps_stream stream) {
  using namespace tps;
  AttnArgs a;
  if (int e = attn_validate("pruned_attn", q_act, k, v, idx, count, cap, N, H, d, scale, blockmask, block, o_act,
                            lse, &a))
    return e;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int e = d == 64 ? launch<64>(a, st) : launch<128>(a, st);
  return e ? e : ok();
}
