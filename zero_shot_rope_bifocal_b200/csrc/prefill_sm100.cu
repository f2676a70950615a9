// prefill_sm100.cu -- bifocal causal attention for a whole prompt on sm_100a.
//
// Method (Jet-Long paper): score rule of §3 (local pairs i - j <= w0 at true
// positions, older pairs at the remapped positions f(i), f(j)), schedule of
// §3.1 (one G for the call), merge of §3.3.  The inclusion-exclusion merge of
// three attention passes equals one softmax whose score for each pair is
// picked by the rule; this kernel runs that single online softmax, visiting
// each key tile with the operand variant(s) its pairs need:
//
//   * a "remote" visit of key tile kt uses (q_remote, k_remote) and keeps only
//     the pairs with i - j > w0;
//   * a "local" visit uses (q_true, k_true) and keeps pairs with
//     0 <= i - j <= w0 (causal).
//
// Tiles that straddle the window edge are visited twice, once per variant,
// each with its complementary mask, so every pair is counted exactly once and
// nothing is subtracted (no cancellation).  For one 128-row query tile the
// remote visits form a prefix of the key tiles and the local visits a suffix,
// so the query operand switches from q_remote to q_true exactly once.  With
// G == 1 (L <= w_pretrained) f is the identity and every tile is a plain
// causal "local" visit: the native-window case of Appendix H.
//
// Operands: the RoPE pass leaves q/k (both variants) and v in the workspace as
// FP16, head-major [B, H, L, D].  FP16 keeps three more mantissa bits than
// BF16 for the rotated values the tensor core must consume in 16 bits.
//
// Hardware mapping (one CTA = one 128-row query tile of one head; 4 warps):
//   * TMA (128-byte swizzle) loads the query tile once per variant and K / V
//     tiles into a two-slot ring; mbarriers with expect-tx track arrival;
//   * thread 0 issues tcgen05.mma: S = Q K^T (M=128, N=128, K=D) into TMEM,
//     later O += P V with P read from TMEM (M=128, N=D, K=128);
//   * every thread owns one query row = one TMEM lane: it loads its S row,
//     applies the mask, runs the online softmax in base 2 (fp32 statistics),
//     rescales its O row only when the running max grew by more than 2^8
//     (decided per warp, since TMEM loads and stores are warp-collective),
//     and stores P (FP16) to TMEM;
//   * the epilogue divides O by the row sum and writes O and the natural-log
//     LSE.
// Each wait is bounded in time (jl::kWaitLimitNs); on expiry the CTA records a
// device error, drains its own MMAs, frees TMEM and exits, and CTAs that start
// after a recorded error skip their work.
#include <cmath>

#include "jl_common.cuh"
#include "sm100_ptx.cuh"

namespace jl {
namespace {

constexpr int BM = 128;  // query rows per tile (= TMEM lanes)
constexpr int BN = 128;  // keys per tile
constexpr int kThreads = 128;
constexpr float kRescaleThreshold = 8.0f;  // log2 units
constexpr uint32_t kF16 = 0;               // operand format code of kind::f16

template <int D>
struct Layout {
  static constexpr int TILE = BM * D * 2;       // bytes of one 128 x D 16-bit tile
  static constexpr int BOX = 128 * 128;         // bytes of one 128-row x 64-col swizzled box
  static constexpr int Q = 0;
  static constexpr int K0 = TILE;
  static constexpr int V0 = 3 * TILE;
  static constexpr int BAR = 5 * TILE;
  static constexpr int BYTES = BAR + 64;
  static constexpr int ALLOC = BYTES + 1024;    // slack to align the base to 1024
  // TMEM columns: S (128) + O (D) + P (64), rounded up to a power of two.
  // D = 128 uses all 512 columns and its shared memory keeps one CTA per SM;
  // D = 64 fits two CTAs per SM in both.
  static constexpr uint32_t TMEM_COLS = D == 128 ? 512u : 256u;
};

struct Params {
  int B, Hq, Hkv, L, G, w0eff, n_qt;
  float scale_log2;
  void *out;
  float *lse;
  int out_f32;
  unsigned int *dev_error;
};

__device__ __forceinline__ float u2f(uint32_t u) { return __uint_as_float(u); }

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
bifocal_prefill_kernel(const __grid_constant__ CUtensorMap tm_qt,
                       const __grid_constant__ CUtensorMap tm_qr,
                       const __grid_constant__ CUtensorMap tm_kt,
                       const __grid_constant__ CUtensorMap tm_kr,
                       const __grid_constant__ CUtensorMap tm_v, const Params prm) {
  using LY = Layout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sb = smem_u32(smem);
  const uint32_t sQ = sb + LY::Q;
  const uint32_t sK[2] = {sb + LY::K0, sb + LY::K0 + LY::TILE};
  const uint32_t sV[2] = {sb + LY::V0, sb + LY::V0 + LY::TILE};
  const uint32_t bar_q = sb + LY::BAR;
  const uint32_t bar_kv[2] = {sb + LY::BAR + 8, sb + LY::BAR + 16};
  const uint32_t bar_s = sb + LY::BAR + 24;
  const uint32_t bar_o = sb + LY::BAR + 32;
  const uint32_t tmem_slot = sb + LY::BAR + 40;
  volatile uint32_t *skip_flag = reinterpret_cast<volatile uint32_t *>(smem + LY::BAR + 44);

  const int tid = threadIdx.x, warp = tid >> 5;
  const int qt = prm.n_qt - 1 - static_cast<int>(blockIdx.x);  // longest rows first
  const int h = blockIdx.y, b = blockIdx.z;
  const int hk = h / (prm.Hq / prm.Hkv);
  const int p0 = qt * BM;
  const int p1 = min(p0 + BM, prm.L) - 1;
  const int row = p0 + tid;
  const bool row_ok = row < prm.L;
  const int w0 = prm.w0eff;

  // Visit plan: remote visits of key tiles [0, n_rem), then local visits of
  // key tiles [kl0, n_kt).  Every causal pair of the tile is kept by exactly
  // one visit.
  const int n_kt = p1 / BN + 1;
  int n_rem = 0, kl0 = 0;
  if (prm.G > 1) {
    n_rem = (p1 - w0 > 0) ? ((p1 - w0 - 1) / BN + 1) : 0;
    kl0 = max(0, p0 - w0) / BN;
  }
  const int nv = n_rem + (n_kt - kl0);

  // Once any CTA has recorded a failure, the others skip their work, so a
  // broken launch ends after one wait limit instead of one per CTA wave.
  // Thread 0 reads the word and the whole CTA follows its answer.
  if (tid == 0) *skip_flag = *reinterpret_cast<volatile unsigned int *>(prm.dev_error);
  __syncthreads();
  if (*skip_flag != kDevOk) return;

  if (tid == 0) {
    mbar_init(bar_q, 1);
    mbar_init(bar_kv[0], 1);
    mbar_init(bar_kv[1], 1);
    mbar_init(bar_s, 1);
    mbar_init(bar_o, 1);
    fence_mbar_init();
    prefetch_tmap(&tm_qt);
    prefetch_tmap(&tm_qr);
    prefetch_tmap(&tm_kt);
    prefetch_tmap(&tm_kr);
    prefetch_tmap(&tm_v);
  }
  __syncthreads();
  if (warp == 0) {
    tmem_alloc(tmem_slot, LY::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(smem + LY::BAR + 40);
  const uint32_t tS = tmem;            // S: 128 columns fp32
  const uint32_t tO = tmem + 128;      // O: D columns fp32
  const uint32_t tP = tmem + 128 + D;  // P: 64 columns of packed FP16 pairs
  const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;

  constexpr uint32_t IDESC_QK = idesc_f16kind_f32(BM, BN, kF16, false, false);
  constexpr uint32_t IDESC_PV = idesc_f16kind_f32(BM, D, kF16, false, true);
  constexpr int NBOX = D / 64;

  auto load_q = [&](bool remote) {
    mbar_arrive_expect_tx(bar_q, LY::TILE);
    for (int c = 0; c < NBOX; ++c)
      tma_load_3d(sQ + c * LY::BOX, remote ? &tm_qr : &tm_qt, bar_q, c * 64, p0, b * prm.Hq + h);
  };
  auto load_kv = [&](int vt, int slot) {
    const bool remote = vt < n_rem;
    const int kt = remote ? vt : kl0 + (vt - n_rem);
    mbar_arrive_expect_tx(bar_kv[slot], 2 * LY::TILE);
    for (int c = 0; c < NBOX; ++c) {
      tma_load_3d(sK[slot] + c * LY::BOX, remote ? &tm_kr : &tm_kt, bar_kv[slot], c * 64, kt * BN,
                  b * prm.Hkv + hk);
      tma_load_3d(sV[slot] + c * LY::BOX, &tm_v, bar_kv[slot], c * 64, kt * BN, b * prm.Hkv + hk);
    }
  };

  if (tid == 0) {
    load_q(n_rem > 0);
    load_kv(0, 0);
  }

  float m_used = -INFINITY;  // reference max of this row (base 2)
  float l_sum = 0.f;
  bool ok = true;

  for (int vt = 0; vt < nv; ++vt) {
    const bool remote = vt < n_rem;
    const int kt = remote ? vt : kl0 + (vt - n_rem);
    const int slot = vt & 1;
    if (tid == 0 && ok) {
      if (vt == 0 || vt == n_rem) ok = mbar_wait_bounded(bar_q, vt == 0 ? 0u : 1u, kWaitLimitNs);
      if (ok)
        ok = mbar_wait_bounded(bar_kv[slot], static_cast<uint32_t>(vt >> 1) & 1u, kWaitLimitNs);
      if (ok) {
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * LY::BOX + (kk & 3) * 32;
          mma_f16kind_ss(tS, smem_desc_sw128(sQ + off, 16, 1024),
                         smem_desc_sw128(sK[slot] + off, 16, 1024), IDESC_QK, kk > 0 ? 1u : 0u);
        }
        mma_commit(bar_s);
      }
    }
    if (ok) ok = mbar_wait_bounded(bar_s, static_cast<uint32_t>(vt) & 1u, kWaitLimitNs);
    if (__syncthreads_or(!ok)) {
      ok = false;
      break;
    }
    tc_fence_after();
    // S(vt) is complete, and with it every earlier MMA: the Q buffer (if this
    // was the last remote visit) and the other K/V slot are free.
    if (tid == 0 && vt + 1 < nv) {
      if (vt + 1 == n_rem) load_q(false);
      load_kv(vt + 1, slot ^ 1);
    }

    // ---- softmax on this thread's row (TMEM accesses are warp-collective:
    // every branch around them below is warp-uniform)
    float x[BN];
    {
      uint32_t r[BN / 32][32];
#pragma unroll
      for (int c = 0; c < BN / 32; ++c) tmem_ld32(tS + lane_base + c * 32, r[c]);
      tmem_wait_ld();
#pragma unroll
      for (int c = 0; c < BN / 32; ++c) {
        reg_fence(r[c]);
#pragma unroll
        for (int e = 0; e < 32; ++e) x[c * 32 + e] = u2f(r[c][e]) * prm.scale_log2;
      }
    }
    const int k0 = kt * BN;
    bool whole;
    if (remote)
      whole = row_ok && (row - (k0 + BN - 1) > w0);
    else
      whole = row_ok && (k0 + BN - 1 <= row) && (row - k0 <= w0);
    if (!whole) {
#pragma unroll
      for (int c = 0; c < BN; ++c) {
        const int d = row - (k0 + c);
        const bool valid = row_ok && d >= 0 && (remote ? (d > w0) : (d <= w0));
        if (!valid) x[c] = -INFINITY;
      }
    }
    float tmax = -INFINITY;
#pragma unroll
    for (int c = 0; c < BN; ++c) tmax = fmaxf(tmax, x[c]);
    const bool grow = tmax > m_used + kRescaleThreshold || (m_used == -INFINITY && tmax > -INFINITY);
    float alpha = 1.f;  // factor applied to this row's O and l
    if (grow) {
      if (m_used != -INFINITY) alpha = exp2f(m_used - tmax);
      m_used = tmax;
    }
    l_sum *= alpha;
    // O holds data from visit 1 on (visit 0 overwrites it); rows whose max was
    // -inf have O = 0 there, so alpha = 1 keeps them exact.
    if (vt > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
      __syncwarp();
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tO + lane_base + c * 32, r);
        tmem_wait_ld();
        reg_fence(r);
#pragma unroll
        for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(u2f(r[e]) * alpha);
        tmem_st32(tO + lane_base + c * 32, r);
      }
    }
    float lsum = 0.f;
    if (m_used == -INFINITY) {
#pragma unroll
      for (int c = 0; c < BN; ++c) x[c] = 0.f;
    } else {
#pragma unroll
      for (int c = 0; c < BN; ++c) {
        x[c] = exp2f(x[c] - m_used);
        lsum += x[c];
      }
    }
    l_sum += lsum;
    __syncwarp();
#pragma unroll
    for (int c = 0; c < BN / 64; ++c) {
      uint32_t r[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const __half2 pr = __floats2half2_rn(x[c * 64 + 2 * e], x[c * 64 + 2 * e + 1]);
        r[e] = *reinterpret_cast<const uint32_t *>(&pr);
      }
      tmem_st32(tP + lane_base + c * 32, r);
    }
    tmem_wait_st();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < BN / 16; ++kk)
        mma_f16kind_ts(tO, tP + kk * 8, smem_desc_sw128(sV[slot] + kk * 16 * 128, LY::BOX, 1024),
                       IDESC_PV, (vt > 0 || kk > 0) ? 1u : 0u);
    }
  }

  // Drain: every MMA issued by thread 0 completes before O is read / TMEM freed.
  if (tid == 0) mma_commit(bar_o);
  const bool drained = mbar_wait_bounded(bar_o, 0u, kWaitLimitNs);
  tc_fence_after();
  const bool good = __syncthreads_and(ok && drained);
  if (!good) {
    if (tid == 0) atomicOr(prm.dev_error, kDevTimeout);
  } else {
    const float inv_l = row_ok ? 1.f / l_sum : 0.f;
    const size_t obase = ((static_cast<size_t>(b) * prm.L + row) * prm.Hq + h) * D;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      uint32_t r[32];
      __syncwarp();
      tmem_ld32(tO + lane_base + c * 32, r);  // whole warp, valid row or not
      tmem_wait_ld();
      reg_fence(r);
      if (!row_ok) continue;
      if (prm.out_f32) {
        float4 *dst = reinterpret_cast<float4 *>(reinterpret_cast<float *>(prm.out) + obase + c * 32);
#pragma unroll
        for (int e = 0; e < 8; ++e)
          dst[e] = make_float4(u2f(r[4 * e]) * inv_l, u2f(r[4 * e + 1]) * inv_l,
                               u2f(r[4 * e + 2]) * inv_l, u2f(r[4 * e + 3]) * inv_l);
      } else {
        uint4 *dst = reinterpret_cast<uint4 *>(reinterpret_cast<__nv_bfloat16 *>(prm.out) + obase + c * 32);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          uint32_t w[4];
#pragma unroll
          for (int f = 0; f < 4; ++f) {
            const __nv_bfloat162 pr = __floats2bfloat162_rn(u2f(r[8 * e + 2 * f]) * inv_l,
                                                            u2f(r[8 * e + 2 * f + 1]) * inv_l);
            w[f] = *reinterpret_cast<const uint32_t *>(&pr);
          }
          dst[e] = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
    }
    if (row_ok && prm.lse)
      prm.lse[(static_cast<size_t>(b) * prm.Hq + h) * prm.L + row] =
          (m_used + log2f(l_sum)) * 0.69314718055994531f;
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, LY::TMEM_COLS);
}

// ---------------------------------------------------------------- host side
using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// Head-major operand [BH, L, D] FP16: box = 64 channels x 128 tokens of one head.
bool encode_head_major(CUtensorMap *tm, const void *base, int BH, int L, int D) {
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(L),
                              static_cast<cuuint64_t>(BH)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2,
                                 static_cast<cuuint64_t>(L) * D * 2};
  const cuuint32_t box[3] = {64, 128, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return encode_fn()(tm, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<void *>(base), dims, strides,
                     box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

template <int D>
cudaError_t launch_d(const PrefillArgs &a, cudaStream_t stream) {
  if (!encode_fn()) return cudaErrorNotSupported;
  CUtensorMap tqt, tqr, tkt, tkr, tv;
  const bool two = a.G > 1;
  if (!encode_head_major(&tqt, a.q_true, a.B * a.Hq, a.L, D) ||
      !encode_head_major(&tqr, two ? a.q_remote : a.q_true, a.B * a.Hq, a.L, D) ||
      !encode_head_major(&tkt, a.k_true, a.B * a.Hkv, a.L, D) ||
      !encode_head_major(&tkr, two ? a.k_remote : a.k_true, a.B * a.Hkv, a.L, D) ||
      !encode_head_major(&tv, a.v_op, a.B * a.Hkv, a.L, D))
    return cudaErrorInvalidValue;
  Params prm;
  prm.B = a.B;
  prm.Hq = a.Hq;
  prm.Hkv = a.Hkv;
  prm.L = a.L;
  prm.G = a.G;
  prm.w0eff = a.G == 1 ? INT_MAX : a.w0;
  prm.n_qt = (a.L + BM - 1) / BM;
  prm.scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(D));
  prm.out = a.out;
  prm.lse = a.lse;
  prm.out_f32 = a.out_f32;
  prm.dev_error = a.dev_error;
  const int smem = Layout<D>::ALLOC;
  cudaError_t e = cudaFuncSetAttribute(bifocal_prefill_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const dim3 grid(prm.n_qt, a.Hq, a.B);
  bifocal_prefill_kernel<D><<<grid, kThreads, smem, stream>>>(tqt, tqr, tkt, tkr, tv, prm);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill_attention(const PrefillArgs &a, cudaStream_t stream) {
  if (a.D == 128) return launch_d<128>(a, stream);
  return launch_d<64>(a, stream);
}

}  // namespace jl
