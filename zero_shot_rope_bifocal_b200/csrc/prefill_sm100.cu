// prefill_sm100.cu -- bifocal causal attention for a whole prompt (or a chunk
// of queries appended to a cache) on sm_100a.
//
// Method (Jet-Long paper): score rule of §3 (local pairs i - j <= w0 at true
// positions, older pairs at the remapped positions f(i), f(j)), schedule of
// §3.1 (one G for the call), merge of §3.3.  The inclusion-exclusion merge of
// three attention passes equals one softmax whose score for each pair is
// picked by the rule; this kernel runs that single online softmax, visiting
// each key tile with the operand variant(s) its pairs need:
//
//   * a "remote" visit of key tile kt uses the query tile rotated to remote
//     positions and k_remote, and keeps only the pairs with i - j > w0;
//   * a "local" visit uses the query tile at true positions and k_true, and
//     keeps pairs with 0 <= i - j <= w0 (causal).
//
// Tiles that straddle the window edge are visited twice, once per variant,
// each with its complementary mask, so every pair is counted exactly once and
// nothing is subtracted (no cancellation).  For one 128-row query tile the
// remote visits form a prefix of the key tiles and the local visits a suffix,
// so the query tile switches from remote to true positions exactly once.
// With G == 1 (L <= w_pretrained) f is the identity and every tile is a plain
// causal "local" visit: the native-window case of Appendix H.
//
// Operands: RoPE runs in the Q load path -- the softmax threads turn the
// BF16 queries into the FP16 query tile in shared memory (build_q_row) -- and
// the key pass leaves k at true and remote positions and v in the workspace
// as FP16, head-major [B, Hkv, L, D], since every key tile is read by every
// query tile of its head.  FP16 keeps three more mantissa bits than BF16 for
// the rotated values the tensor core must consume in 16 bits.
//
// CTA = two 128-row query tiles of the same 128 positions, for two query
// heads of one KV group (GQA packing: each K/V tile staged in shared memory
// serves 256 query rows).  Warp-specialised, 10 warps:
//   * warps 0-3 / 4-7: softmax for query tile 0 / 1, one thread per row (a
//     TMEM lane).  A thread builds its row of the query tile, holds its row's
//     128 scores in registers: one TMEM read, the row max, the exponentials,
//     P stored back, with no exchange between threads; it rescales its O row
//     when the max grows and runs the epilogue of its row;
//   * warp 8: TMA producer of the K and V tiles through a ring of two
//     two-tile units, unit u holding V(u-1) and K(u): the pair the MMA
//     issuer uses in the same visit, so one wait and one release per visit;
//   * warp 9: tcgen05.mma issuer, in the order
//       S0(j+1) = Q0 K(j+1)^T after O0 += P0(j) V(j), and likewise for tile 1,
//     so the tensor core works on one tile while the other tile's softmax
//     runs.
// Ten warps put three on two of the four SM sub-partitions, whose register
// files then allow 168 registers per thread: enough for a whole row.
// TMEM (512 columns): S0 | S1 | O0 | O1; a row's P (packed FP16) is written
// over the first 64 columns of its S once the scores are in registers.
// A chunk with few query tiles splits each tile's visit list into contiguous
// ranges, one CTA each (grid z): such a CTA writes its rows' unnormalised O
// with the running max and sum, and a log-sum-exp merge kernel forms the
// output (launch_split_merge).
// Each wait is bounded in time (jl::kWaitLimitNs) and also gives up when
// another role has given up; the CTA then records a device error, drains its
// MMAs and in-flight copies, frees TMEM and exits.
#include <cmath>

#include "jl_common.cuh"
#include "sm100_ptx.cuh"

namespace jl {
namespace {

constexpr int BM = 128;  // query rows per tile (= TMEM lanes)
constexpr int BN = 128;  // keys per tile
constexpr int NU = 2;    // K/V ring units of two tiles: unit u = V(u-1), K(u)
constexpr int kSoftmaxWarps = 8;  // 2 warpgroups: one per query tile
constexpr int kWarps = 10;
constexpr int kThreads = kWarps * 32;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
// Column pairs per 8 whose exponential runs on the FMA pipe (the rest on the
// special-function unit, which would otherwise be the softmax's limit).
#ifndef JL_PREFILL_FMA_PAIRS
#define JL_PREFILL_FMA_PAIRS 1
#endif
constexpr int kFmaPairsPer8 = JL_PREFILL_FMA_PAIRS;
constexpr float kRescaleThreshold = 8.0f;  // log2 units
constexpr uint32_t kF16 = 0;               // operand format code of kind::f16

template <int D>
struct Layout {
  static constexpr int TILE = BM * D * 2;  // bytes of one 128 x D FP16 tile
  static constexpr int BOX = 128 * 128;    // bytes of one 128-row x 64-col swizzled box
  static constexpr int Q0 = 0;
  static constexpr int RING = 2 * TILE;
  static constexpr int BAR = RING + 2 * NU * TILE;
  // barrier indices (8 bytes each)
  static constexpr int kQFull = 0, kKvFull = 4, kKvEmpty = 4 + NU,
                       kSFull = 4 + 2 * NU, kPFull = 6 + 2 * NU, kOFull = 8 + 2 * NU,
                       kDrain = 10 + 2 * NU, kNumBars = 11 + 2 * NU;
  static constexpr int TMEM_SLOT = BAR + 8 * kNumBars;
  static constexpr int ABORT = TMEM_SLOT + 4;
  static constexpr int SKIP = TMEM_SLOT + 8;
  static constexpr int BYTES = TMEM_SLOT + 16;
  // 1024 B of slack to align the base; D = 64 asks for enough shared memory
  // to keep one CTA per SM, since each CTA holds all 512 TMEM columns.
  static constexpr int ALLOC = (BYTES + 1024 > 120 * 1024) ? BYTES + 1024 : 120 * 1024;
};

struct Params {
  // query rows are positions [q_off, q_off + Lq) (a whole prompt: q_off = 0,
  // Lq = L; a chunk appended to a cache: q_off = P0); keys are [0, q_off + Lq)
  int B, Hq, Hkv, q_off, Lq, G, w0eff, n_qt, grp, npair;
  int pass;  // PrefillPass: the fused rule or one pass of the three-pass merge
  float scale_log2;
  // Queries, pre-RoPE BF16 [B, Lq, Hq, D]: the softmax threads rotate their
  // rows into the FP16 operand tiles.  omega[i] = theta_i / (2 pi), turns per
  // position as a 64-bit binary fraction; omega_remote[i] is the remote
  // map's (theta_i, or theta'_i under the frequency interpolation, where the
  // remote position is the true one).
  const __nv_bfloat16 *q_raw;
  int remote_interp;
  uint64_t omega[64], omega_remote[64];
  void *out;
  float *lse;
  int out_f32;
  unsigned int *dev_error;
  // key split: blockIdx.z = b * n_split + split; with n_split > 1 each CTA
  // takes a contiguous share of its tile's visits and writes partial
  // records [B, Lq, Hq, n_split, D + 2] (O unnormalised, m in base 2, l)
  int n_split;
  float *partial;
};

__device__ __forceinline__ float u2f(uint32_t u) { return __uint_as_float(u); }

// 2^x on the FMA pipe for a pair of arguments (x <= 2^22), used for a share
// of the softmax exponentials so that the special-function unit is not the
// bottleneck.  x = n + f with n = round(x), f in [-1/2, 1/2]; 2^f is a cubic
// whose coefficients come from exp2_poly_fit.py (relative error 7.5e-5,
// below the FP16 rounding of P); 2^n is added to the exponent field.
// Arguments are clamped at -125, so -inf gives 2^-125 (zero once in FP16).
__device__ __forceinline__ float2 exp2_fma2(float2 x) {
  constexpr float kRound = 12582912.0f;  // 1.5 * 2^23: x + kRound rounds x to an integer
  x.x = fmaxf(x.x, -125.0f);
  x.y = fmaxf(x.y, -125.0f);
  const float2 t = fadd2(x, make_float2(kRound, kRound));      // n in the low mantissa bits
  const float2 n = fadd2(t, make_float2(-kRound, -kRound));    // n as a float
  const float2 f = ffma2(n, make_float2(-1.f, -1.f), x);       // x - n
  float2 p = ffma2(make_float2(0.0551716648f, 0.0551716648f), f,
                   make_float2(0.242611125f, 0.242611125f));
  p = ffma2(p, f, make_float2(0.693260968f, 0.693260968f));
  p = ffma2(p, f, make_float2(0.999928057f, 0.999928057f));
  // bits(t) << 23 == n << 23 (the bits of kRound shift out); add to p's exponent
  return make_float2(__int_as_float(__float_as_int(p.x) + (__float_as_int(t.x) << 23)),
                     __int_as_float(__float_as_int(p.y) + (__float_as_int(t.y) << 23)));
}

// Bounded wait that also gives up once another role has raised `abort`.
__device__ __forceinline__ bool wait_or_abort(uint32_t bar, uint32_t parity,
                                              volatile uint32_t *abort) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 0u) {
      if (*abort) return false;
      if (global_timer_ns() - t0 > kWaitLimitNs) {
        *abort = 1u;
        return false;
      }
    }
  }
}

// RoPE in the Q load path: one softmax thread turns its row of the query
// into the FP16 operand tile of its query tile, at the remote position
// (f(row), or row with the remote map's frequencies) or at the true
// position.  The tile is 128-byte swizzled as the MMA descriptors expect:
// row r of a 64-channel box is 128 bytes, its 16-byte chunk k stored at chunk
// k ^ (r % 8).  Rows past the last query are zero.  The angle pos * theta_i
// is exact modulo one turn: the wrapping 64-bit product with theta_i / (2 pi)
// (a 64-bit binary fraction) has the signed phase in its top 32 bits, so the
// sine/cosine only sees [-pi, pi).  The generic-proxy writes are fenced for
// the async proxy before the caller's arrival on the tile's barrier.  Kept out
// of line: it runs twice per CTA and its registers stay out of the visit loop.
template <int D>
__device__ __noinline__ void build_q_row(uint8_t *tile, int rloc, int row, bool row_ok, int b,
                                         int head, bool remote_var, const Params &prm) {
  constexpr int BOX = 128 * 128;
  auto store16 = [&](int c, uint4 v) {  // channels [c, c + 8)
    uint8_t *box = tile + (c >> 6) * BOX + rloc * 128;
    *reinterpret_cast<uint4 *>(box + ((((c & 63) >> 3) ^ (rloc & 7)) << 4)) = v;
  };
  bool in_range = true;
  if (row_ok) {
    const uint64_t pos =
        static_cast<uint64_t>((!remote_var || prm.remote_interp) ? row : remap(row, prm.G));
    const uint64_t *om = remote_var ? prm.omega_remote : prm.omega;
    constexpr float kTurnToRad = 1.4629180792671596e-09f;  // 2 pi / 2^32
    auto cos_sin = [&](int i, float &cv, float &sv) {
      const int32_t ph = static_cast<int32_t>((pos * om[i]) >> 32);
      __sincosf(static_cast<float>(ph) * kTurnToRad, &sv, &cv);
    };
    const uint4 *src = reinterpret_cast<const uint4 *>(
        prm.q_raw + ((static_cast<size_t>(b) * prm.Lq + (row - prm.q_off)) * prm.Hq + head) * D);
    uint4 raw[D / 8];  // the whole row, all loads in flight at once
#pragma unroll
    for (int k = 0; k < D / 8; ++k) raw[k] = __ldg(src + k);
#pragma unroll
    for (int c = 0; c < D / 2; c += 8) {  // channels c.. and their partners c + D/2..
      const uint4 xa = raw[c / 8], xb = raw[(c + D / 2) / 8];
      const uint32_t wa[4] = {xa.x, xa.y, xa.z, xa.w}, wb[4] = {xb.x, xb.y, xb.z, xb.w};
      uint32_t oa[4], ob[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float c0, s0, c1, s1;
        cos_sin(c + 2 * e, c0, s0);
        cos_sin(c + 2 * e + 1, c1, s1);
        const float x0 = __uint_as_float(wa[e] << 16), x1 = __uint_as_float(wa[e] & 0xffff0000u);
        const float y0 = __uint_as_float(wb[e] << 16), y1 = __uint_as_float(wb[e] & 0xffff0000u);
        const __half2 lo = __floats2half2_rn(x0 * c0 - y0 * s0, x1 * c1 - y1 * s1);
        const __half2 hi = __floats2half2_rn(x0 * s0 + y0 * c0, x1 * s1 + y1 * c1);
        in_range &= !(__hisinf(__low2half(lo)) | __hisinf(__high2half(lo)) |
                      __hisinf(__low2half(hi)) | __hisinf(__high2half(hi)));
        oa[e] = *reinterpret_cast<const uint32_t *>(&lo);
        ob[e] = *reinterpret_cast<const uint32_t *>(&hi);
      }
      store16(c, make_uint4(oa[0], oa[1], oa[2], oa[3]));
      store16(c + D / 2, make_uint4(ob[0], ob[1], ob[2], ob[3]));
    }
  } else {
#pragma unroll
    for (int c = 0; c < D; c += 8) store16(c, make_uint4(0u, 0u, 0u, 0u));
  }
  if (!in_range) atomicOr(prm.dev_error, kDevRange);
  fence_proxy_async_smem();
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
bifocal_prefill_kernel(const __grid_constant__ CUtensorMap tm_kt,
                       const __grid_constant__ CUtensorMap tm_kr,
                       const __grid_constant__ CUtensorMap tm_v,
                       const __grid_constant__ Params prm) {
  using LY = Layout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sb = smem_u32(smem);
  auto bar = [&](int i) { return sb + LY::BAR + 8u * static_cast<uint32_t>(i); };
  volatile uint32_t *abort = reinterpret_cast<volatile uint32_t *>(smem + LY::ABORT);
  volatile uint32_t *skip = reinterpret_cast<volatile uint32_t *>(smem + LY::SKIP);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qt = prm.n_qt - 1 - static_cast<int>(blockIdx.x);  // longest rows first
  const int g = static_cast<int>(blockIdx.y) / prm.npair;
  const int pr = static_cast<int>(blockIdx.y) - g * prm.npair;
  const int split = static_cast<int>(blockIdx.z) % prm.n_split;
  const int b = static_cast<int>(blockIdx.z) / prm.n_split;
  const int head0 = g * prm.grp + 2 * pr;
  const bool has1 = 2 * pr + 1 < prm.grp;
  const int p0 = prm.q_off + qt * BM;  // position of the tile's first row
  const int p1 = min(p0 + BM, prm.q_off + prm.Lq) - 1;
  const int w0 = prm.w0eff;

  // Visit plan: remote visits of key tiles [kr0, kr0 + n_rem), then local
  // visits of key tiles [kl0, n_kt).  A remote visit keeps the pairs with
  // dlo <= i - j <= dhi, a local visit those with 0 <= i - j <= w0.  Fused
  // rule: remote tiles [0, n_rem) with i - j > w0, so every causal pair of
  // the tile is kept by exactly one visit.  The passes of the three-pass
  // merge (§3.3) reuse the same machinery: A = remote positions on every
  // causal pair, B = true positions on the band 0 <= i - j <= w0, C = remote
  // positions on the band.
  const int n_kt = p1 / BN + 1;
  int n_rem = 0, kl0 = 0, kr0 = 0;
  int dlo = w0 == INT_MAX ? INT_MAX : w0 + 1, dhi = INT_MAX;
  if (prm.pass == kPassFused) {
    if (prm.G > 1) {
      n_rem = (p1 - w0 > 0) ? ((p1 - w0 - 1) / BN + 1) : 0;
      kl0 = max(0, p0 - w0) / BN;
    }
  } else if (prm.pass == kPassRemoteCausal) {
    n_rem = n_kt;
    kl0 = n_kt;
    dlo = 0;
  } else if (prm.pass == kPassLocalBand) {
    kl0 = max(0, p0 - w0) / BN;
  } else {  // kPassRemoteBand
    kr0 = max(0, p0 - w0) / BN;
    n_rem = n_kt - kr0;
    kl0 = n_kt;
    dlo = 0;
    dhi = w0;
  }
  int nv = n_rem + (n_kt - kl0);
  if (prm.n_split > 1) {
    // This split's share [v0, v1) of the visits: a remote part (if it
    // starts before the local visits) and a local part, in the same order.
    const int v0 = static_cast<int>(static_cast<long long>(nv) * split / prm.n_split);
    const int v1 = static_cast<int>(static_cast<long long>(nv) * (split + 1) / prm.n_split);
    if (v0 < n_rem) {
      kr0 += v0;
      n_rem = min(n_rem, v1) - v0;
    } else {
      kl0 += v0 - n_rem;
      n_rem = 0;
    }
    nv = v1 - v0;
  }
  const bool switch_q = n_rem > 0 && n_rem < nv;

  // A launch that already recorded a failure ends quickly: thread 0 reads the
  // error word and the whole CTA follows its answer.
  if (tid == 0) {
    *skip = *reinterpret_cast<volatile unsigned int *>(prm.dev_error);
    *abort = 0u;
  }
  __syncthreads();
  if (*skip != kDevOk) return;

  if (tid == 0) {
    // Q-ready and P-ready barriers take one arrival from every softmax
    // thread of the tile (one per row); all others one arrival (plus
    // transaction bytes for TMA).
    for (int i = 0; i < LY::kNumBars; ++i)
      mbar_init(bar(i), (i == LY::kPFull || i == LY::kPFull + 1 || i == LY::kQFull ||
                         i == LY::kQFull + 1)
                            ? BM
                            : 1);
    fence_mbar_init();
  }
  if (warp == kProducerWarp && lane == 0) {
    prefetch_tmap(&tm_kt);
    prefetch_tmap(&tm_kr);
    prefetch_tmap(&tm_v);
  }
  __syncthreads();
  if (warp == kMmaWarp) {
    tmem_alloc(sb + LY::TMEM_SLOT, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(smem + LY::TMEM_SLOT);
  // TMEM columns: S0 [0,128) S1 [128,256) O0 [256,256+D) O1 [256+D,256+2D)
  auto tS = [&](int s) { return tmem + 128u * static_cast<uint32_t>(s); };
  auto tO = [&](int s) { return tmem + 256u + static_cast<uint32_t>(D * s); };

  constexpr uint32_t IDESC_QK = idesc_f16kind_f32(BM, BN, kF16, false, false);
  constexpr uint32_t IDESC_PV = idesc_f16kind_f32(BM, D, kF16, false, true);
  constexpr int NBOX = D / 64;

  if (warp >= kSoftmaxWarps) {
    if (warp == kProducerWarp && lane == 0) {
      // ---------------------------------------------------------- producer
      // Unit u holds V(u-1) in its first tile and K(u) in its second (unit 0
      // only K(0), unit nv only V(nv-1)): the pair the MMA issuer uses
      // together in visit u-1 (O += P V(u-1), then S = Q K(u)^T).
      bool ok = true;
      uint32_t issued[NU] = {0, 0};  // uses issued per unit slot
      for (int u = 0; u <= nv && ok; ++u) {
        const int slot = u % NU;
        const uint32_t use = static_cast<uint32_t>(u / NU);
        ok = wait_or_abort(bar(LY::kKvEmpty + slot), (use & 1u) ^ 1u, abort);
        if (!ok) break;
        const uint32_t dst = sb + LY::RING + slot * 2 * LY::TILE;
        const bool has_v = u > 0, has_k = u < nv;
        mbar_arrive_expect_tx(bar(LY::kKvFull + slot), (has_v + has_k) * LY::TILE);
        auto kt_of = [&](int visit) {
          return visit < n_rem ? kr0 + visit : kl0 + (visit - n_rem);
        };
        if (has_v)
          for (int c = 0; c < NBOX; ++c)
            tma_load_3d(dst + c * LY::BOX, &tm_v, bar(LY::kKvFull + slot), c * 64,
                        kt_of(u - 1) * BN, b * prm.Hkv + g);
        if (has_k) {
          const CUtensorMap *tm = u < n_rem ? &tm_kr : &tm_kt;
          for (int c = 0; c < NBOX; ++c)
            tma_load_3d(dst + LY::TILE + c * LY::BOX, tm, bar(LY::kKvFull + slot), c * 64,
                        kt_of(u) * BN, b * prm.Hkv + g);
        }
        issued[slot] = use + 1;
      }
      if (!ok) {
        // Let copies already in flight land before the CTA exits (bounded).
        for (int s = 0; s < NU; ++s)
          if (issued[s] > 0) mbar_wait_bounded(bar(LY::kKvFull + s), (issued[s] - 1u) & 1u, kWaitLimitNs);
      }
    } else if (warp == kMmaWarp && lane == 0) {
      // ---------------------------------------------------------- MMA issuer
      auto qk = [&](int s, uint32_t kaddr) {
        // descriptors of k-step 0; step kk moves the start address by off(kk)
        // (the address field holds addr >> 4 in its low bits)
        const uint64_t dq = smem_desc_sw128(sb + LY::Q0 + s * LY::TILE, 16, 1024);
        const uint64_t dk = smem_desc_sw128(kaddr, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t off = static_cast<uint64_t>(((kk >> 2) * LY::BOX + (kk & 3) * 32) >> 4);
          mma_f16kind_ss(tS(s), dq + off, dk + off, IDESC_QK, kk > 0 ? 1u : 0u);
        }
        mma_commit(bar(LY::kSFull + s));
      };
      auto pv = [&](int s, uint32_t vaddr, bool acc) {
        const uint64_t dv = smem_desc_sw128(vaddr, LY::BOX, 1024);
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk)  // P of keys [16kk, 16kk+16): columns [8kk, 8kk+8)
          mma_f16kind_ts(tO(s), tS(s) + kk * 8,
                         dv + static_cast<uint64_t>((kk * 16 * 128) >> 4), IDESC_PV,
                         (acc || kk > 0) ? 1u : 0u);
      };
      auto unit_addr = [&](int u) { return sb + LY::RING + (u % NU) * 2 * LY::TILE; };
      auto unit_wait = [&](int u) {
        return wait_or_abort(bar(LY::kKvFull + u % NU), static_cast<uint32_t>(u / NU) & 1u, abort);
      };
      bool ok = wait_or_abort(bar(LY::kQFull + 0), 0u, abort);
      if (ok && has1) ok = wait_or_abort(bar(LY::kQFull + 1), 0u, abort);
      // visit 0: S0, S1 from unit 0 (K(0))
      if (ok) ok = unit_wait(0);
      if (ok) {
        tc_fence_after();
        qk(0, unit_addr(0) + LY::TILE);
        if (has1) qk(1, unit_addr(0) + LY::TILE);
        mma_commit(bar(LY::kKvEmpty + 0));
      }
      for (int j = 0; j < nv && ok; ++j) {
        // unit j+1: V(j) and (if more) K(j+1)
        ok = unit_wait(j + 1);
        if (!ok) break;
        const uint32_t va = unit_addr(j + 1), ka = va + LY::TILE;
        // tile 0: O0 += P0(j) V(j), then S0(j+1)
        ok = wait_or_abort(bar(LY::kPFull + 0), static_cast<uint32_t>(j) & 1u, abort);
        if (!ok) break;
        tc_fence_after();
        pv(0, va, j > 0);
        const bool more = j + 1 < nv;
        if (more) {
          if (switch_q && j + 1 == n_rem) ok = wait_or_abort(bar(LY::kQFull + 0), 1u, abort);
          if (!ok) break;
          tc_fence_after();
          qk(0, ka);
        }
        // tile 1: O1 += P1(j) V(j), then S1(j+1)
        if (has1) {
          ok = wait_or_abort(bar(LY::kPFull + 1), static_cast<uint32_t>(j) & 1u, abort);
          if (!ok) break;
          tc_fence_after();
          pv(1, va, j > 0);
          if (more) {
            if (switch_q && j + 1 == n_rem) ok = wait_or_abort(bar(LY::kQFull + 1), 1u, abort);
            if (!ok) break;
            tc_fence_after();
            qk(1, ka);
          }
        }
        mma_commit(bar(LY::kKvEmpty + (j + 1) % NU));
      }
      if (ok) {
        mma_commit(bar(LY::kOFull + 0));
        if (has1) mma_commit(bar(LY::kOFull + 1));
      }
      // Every MMA issued here completes before TMEM is read out or freed.
      mma_commit(bar(LY::kDrain));
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(bar(LY::kDrain), 0u))
        if (global_timer_ns() - t0 > kWaitLimitNs) {
          *abort = 1u;
          break;
        }
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int s = warp >> 2;             // query tile of this warpgroup
    const int wq = warp & 3;             // TMEM lane quarter
    const int rloc = tid & (BM - 1);     // row inside the tile
    const int row = p0 + rloc;
    const bool active = s == 0 || has1;
    const bool row_ok = active && row < prm.q_off + prm.Lq;
    const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
    // RoPE in the Q load path (build_q_row): at the remote position first
    // (if the tile has remote visits), at the true position after the switch.
    auto build_q = [&](bool remote_var) {
      build_q_row<D>(smem + Layout<D>::Q0 + s * Layout<D>::TILE, rloc, row, row_ok, b, head0 + s,
                     remote_var, prm);
      mbar_arrive(bar(LY::kQFull + s));
    };
    if (active) build_q(n_rem > 0);

    float m_used = -INFINITY;  // reference max of this row (base 2)
    float l_sum = 0.f;         // running row sum, relative to m_used
    bool ok = active;
    for (int j = 0; j < nv && ok; ++j) {
      const bool remote = j < n_rem;
      const int kt = remote ? kr0 + j : kl0 + (j - n_rem);
      ok = wait_or_abort(bar(LY::kSFull + s), static_cast<uint32_t>(j) & 1u, abort);
      if (__any_sync(0xffffffffu, !ok)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int k0 = kt * BN;  // key of column 0
      // Rows past the last query (a partial tile) are never written; their
      // scores are finite (their query rows were zero-filled), so they skip
      // the mask like rows whose every pair is kept.
      bool whole = !row_ok;
      if (row_ok && remote)
        whole = (row - (k0 + BN - 1) >= dlo) && (row - k0 <= dhi);
      else if (row_ok)
        whole = (k0 + BN - 1 <= row) && (row - k0 <= w0);
      // The row's raw scores (the scale is positive and applied later), one
      // TMEM read of all 128 columns, then the mask on edge tiles only.
      float x[BN];
      {
        uint32_t(&xr)[BN / 32][32] = reinterpret_cast<uint32_t(&)[BN / 32][32]>(x);
#pragma unroll
        for (int cc = 0; cc < BN / 32; ++cc) tmem_ld32(tS(s) + lane_base + cc * 32, xr[cc]);
        tmem_wait_ld();
#pragma unroll
        for (int cc = 0; cc < BN / 32; ++cc) reg_fence(xr[cc]);
      }
      if (!whole) {
#pragma unroll
        for (int c = 0; c < BN; ++c) {
          const int d = row - (k0 + c);
          const bool valid = row_ok && d >= 0 && (remote ? (d >= dlo && d <= dhi) : (d <= w0));
          if (!valid) x[c] = -INFINITY;
        }
      }
      // row max: four chains of three-input maxima
      float mx[4] = {x[0], x[1], x[2], x[3]};
#pragma unroll
      for (int c = 4; c < BN; c += 8) {
        mx[0] = fmax3(mx[0], x[c], x[c + 1]);
        mx[1] = fmax3(mx[1], x[c + 2], x[c + 3]);
        if (c + 4 < BN) {
          mx[2] = fmax3(mx[2], x[c + 4], x[c + 5]);
          mx[3] = fmax3(mx[3], x[c + 6], x[c + 7]);
        }
      }
      const float tmax = fmax3(fmax3(mx[0], mx[1], mx[2]), mx[3], mx[3]) * prm.scale_log2;
      const bool grow =
          tmax > m_used + kRescaleThreshold || (m_used == -INFINITY && tmax > -INFINITY);
      float alpha = 1.f;
      if (grow) {
        if (m_used != -INFINITY) alpha = exp2f(m_used - tmax);
        m_used = tmax;
      }
      l_sum *= alpha;
      // p = 2^(s * scale - m), written back as packed FP16 P over the first
      // 64 columns in one store (all scores are already in registers).
      // Masked entries are -inf and give 0 (or 2^-125 on the FMA path, which
      // rounds to 0 in FP16); a row with nothing valid yet has all entries
      // -inf.  kFmaPairsPer8 column pairs in eight take the FMA-pipe
      // exponential, the rest the special-function unit.
      const float neg_m = m_used == -INFINITY ? 0.f : -m_used;
      const float2 sc2 = make_float2(prm.scale_log2, prm.scale_log2);
      const float2 nm2 = make_float2(neg_m, neg_m);
      float2 acc2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
      uint32_t pr[BN / 2];
#pragma unroll
      for (int c = 0; c < BN; c += 2) {
        float2 v = ffma2(make_float2(x[c], x[c + 1]), sc2, nm2);
        if (((c >> 1) & 7) < kFmaPairsPer8) {
          v = exp2_fma2(v);
        } else {
          v.x = ex2_sfu(v.x);
          v.y = ex2_sfu(v.y);
        }
        acc2[(c >> 1) & 1] = fadd2(acc2[(c >> 1) & 1], v);
        const __half2 h2 = __floats2half2_rn(v.x, v.y);
        pr[c >> 1] = *reinterpret_cast<const uint32_t *>(&h2);
      }
      tmem_st64(tS(s) + lane_base, pr);
      tmem_wait_st();
      const float2 a = fadd2(acc2[0], acc2[1]);
      l_sum += a.x + a.y;
      // O of this tile holds visits 0..j-1 (all complete: S(j) was issued
      // after P(j-1) V(j-1)); rows whose max was -inf hold 0 there.  The row
      // is rescaled before PV(j) may start.
      if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {  // one 32-column chunk at a time
          uint32_t rr[32];
          const uint32_t col = tO(s) + lane_base + c * 32;
          tmem_ld32(col, rr);
          tmem_wait_ld();
          reg_fence(rr);
#pragma unroll
          for (int e = 0; e < 32; ++e) rr[e] = __float_as_uint(u2f(rr[e]) * alpha);
          tmem_st32(col, rr);
        }
        tmem_wait_st();
      }
      tc_fence_before();
      mbar_arrive(bar(LY::kPFull + s));
      // After the last remote visit the query tile switches to true
      // positions: S(j) was read, so QK(j) is done with the tile.
      if (switch_q && j == n_rem - 1) build_q(false);
    }
    // ---- epilogue: O / l and the log-sum-exp of this row, or (key split)
    // the row's partial record
    if (ok) ok = wait_or_abort(bar(LY::kOFull + s), 0u, abort);
    if (__all_sync(0xffffffffu, ok)) {
      tc_fence_after();
      const float inv_l = row_ok ? 1.f / l_sum : 0.f;
      const int head = head0 + s;
      const size_t row_head = (static_cast<size_t>(b) * prm.Lq + qt * BM + rloc) * prm.Hq + head;
      const size_t obase = row_head * D;
      const bool split_rec = prm.n_split > 1;
      float *rec = split_rec ? prm.partial + (row_head * prm.n_split + split) * (D + 2) : nullptr;
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t rr[32];
        __syncwarp();
        tmem_ld32(tO(s) + lane_base + c * 32, rr);  // whole warp, valid row or not
        tmem_wait_ld();
        reg_fence(rr);
        if (!row_ok) continue;
        if (split_rec) {
          // a split without visits (never planned) has no O in TMEM: zeros
          float2 *dst = reinterpret_cast<float2 *>(rec + c * 32);
#pragma unroll
          for (int e = 0; e < 16; ++e)
            dst[e] = nv > 0 ? make_float2(u2f(rr[2 * e]), u2f(rr[2 * e + 1])) : make_float2(0.f, 0.f);
        } else if (prm.out_f32) {
          float4 *dst = reinterpret_cast<float4 *>(reinterpret_cast<float *>(prm.out) + obase + c * 32);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            dst[e] = make_float4(u2f(rr[4 * e]) * inv_l, u2f(rr[4 * e + 1]) * inv_l,
                                 u2f(rr[4 * e + 2]) * inv_l, u2f(rr[4 * e + 3]) * inv_l);
        } else {
          uint4 *dst = reinterpret_cast<uint4 *>(reinterpret_cast<__nv_bfloat16 *>(prm.out) + obase + c * 32);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            uint32_t wv[4];
#pragma unroll
            for (int f = 0; f < 4; ++f) {
              const __nv_bfloat162 h2 = __floats2bfloat162_rn(u2f(rr[8 * e + 2 * f]) * inv_l,
                                                              u2f(rr[8 * e + 2 * f + 1]) * inv_l);
              wv[f] = *reinterpret_cast<const uint32_t *>(&h2);
            }
            dst[e] = make_uint4(wv[0], wv[1], wv[2], wv[3]);
          }
        }
      }
      if (row_ok && split_rec) {
        rec[D] = m_used;
        rec[D + 1] = l_sum;
      } else if (row_ok && prm.lse) {
        prm.lse[(static_cast<size_t>(b) * prm.Hq + head) * prm.Lq + qt * BM + rloc] =
            (m_used + log2f(l_sum)) * 0.69314718055994531f;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (tid == 0 && *abort) atomicOr(prm.dev_error, kDevTimeout);
  if (warp == kMmaWarp) tmem_dealloc(tmem, 512);
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
  CUtensorMap tkt, tkr, tv;
  const bool two = a.G > 1;
  if (!encode_head_major(&tkt, a.k_true, a.B * a.Hkv, a.L, D) ||
      !encode_head_major(&tkr, two ? a.k_remote : a.k_true, a.B * a.Hkv, a.L, D) ||
      !encode_head_major(&tv, a.v_op, a.B * a.Hkv, a.L, D))
    return cudaErrorInvalidValue;
  Params prm;
  prm.B = a.B;
  prm.Hq = a.Hq;
  prm.Hkv = a.Hkv;
  prm.q_off = a.q_off;
  prm.Lq = a.Lq;
  prm.G = a.G;
  // The fused rule with G = 1 is plain causal attention; a pass of the
  // three-pass merge keeps its band whatever G is.
  prm.w0eff = (a.G == 1 && a.pass == kPassFused) ? INT_MAX : a.w0;
  prm.pass = a.pass;
  prm.n_qt = (a.Lq + BM - 1) / BM;
  prm.grp = a.Hq / a.Hkv;
  prm.npair = (prm.grp + 1) / 2;
  prm.scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(D));
  prm.out = a.out;
  prm.lse = a.lse;
  prm.out_f32 = a.out_f32;
  prm.dev_error = a.dev_error;
  prm.n_split = a.n_split > 1 ? a.n_split : 1;
  prm.partial = a.partial;
  prm.q_raw = a.q;
  prm.remote_interp = a.interp;
  const double log_theta = std::log(static_cast<double>(a.theta));
  const double turns_q64 = 0.15915494309189533577 * 18446744073709551616.0;  // 2^64 / (2 pi)
  for (int i = 0; i < D / 2; ++i) {
    const double f = std::exp(-2.0 * static_cast<double>(i) / static_cast<double>(D) * log_theta);
    const double fr =
        a.interp ? f * interp_factor(f, a.L, a.w_pretrained, a.ramp_alpha, a.ramp_beta) : f;
    prm.omega[i] = static_cast<uint64_t>(std::llround(f * turns_q64));  // < 2^62
    prm.omega_remote[i] = static_cast<uint64_t>(std::llround(fr * turns_q64));
  }
  const int smem = Layout<D>::ALLOC;
  cudaError_t e = ensure_smem_limit<bifocal_prefill_kernel<D>>(smem);
  if (e != cudaSuccess) return e;
  const dim3 grid(prm.n_qt, a.Hkv * prm.npair, a.B * prm.n_split);
  bifocal_prefill_kernel<D><<<grid, kThreads, smem, stream>>>(tkt, tkr, tv, prm);
  e = cudaGetLastError();
  if (e != cudaSuccess || prm.n_split == 1) return e;
  return launch_split_merge(a.partial, prm.n_split, a.out, a.out_f32, a.lse, a.B, a.Lq, a.Hq, D,
                            stream);
}

}  // namespace

cudaError_t launch_prefill_attention(const PrefillArgs &a, cudaStream_t stream) {
  if (a.D == 128) return launch_d<128>(a, stream);
  return launch_d<64>(a, stream);
}

}  // namespace jl
