// decode_kernels.cu -- one generation step of bifocal attention on the
// true-position KV cache (Jet-Long paper, §3.2 "Key-value cache management and
// correction rotation"; score rule of §3; schedule of §3.1 with L = tokens in
// the cache including the new one, query at p = L - 1).
//
// Per token j: keys with p - j <= w0 are scored as cached against
// RoPE(x_q, p); older keys are first turned by the correction rotation
// R(Delta j), Delta j = f(j) - j (so the cache is never rewritten), and scored
// against RoPE(x_q, f(p)).
//
// Split-KV: CTA (s, c, b) streams key chunk s of KV heads [8c, 8c + 8) of
// batch b (two CTAs per SM).  Warp 0 fills a three-stage shared-memory ring
// with bulk async copies (cp.async.bulk, one per token and tensor, into rows
// padded by 16 bytes; completion on the stage's "full" mbarrier).  For each
// stage with remote tokens the CTA also builds a table of
// cos/sin(Delta j * theta_i) for its tokens, shared by all heads; every warp
// writes some of its rows once it is two stages behind.  The phase
// Delta j * theta_i / (2 pi) is formed exactly modulo one turn in 64-bit
// fixed point (theta_i / (2 pi) held as a 64-bit binary fraction), so the
// hardware sine/cosine only ever sees [-pi, pi).
// Eight warps, one per KV head, run each stage on the tensor cores
// (mma.sync m16n8k16):
//   * S = Q K^T: the A operand holds the group's query heads (rows), FP16,
//     pre-scaled by log2(e)/sqrt(D); K arrives through ldmatrix as B
//     fragments, turned (remote tokens, packed FP32x2 arithmetic) and
//     converted to FP16 in registers;
//   * an online softmax per head over the stage's tokens (fp32 statistics,
//     lazy rescaling);
//   * O^T += V^T P^T: V through ldmatrix.trans, P taken straight from the S
//     accumulator fragment (BF16), O^T accumulated in fp32 registers.
// Each warp then releases the stage on its "empty" mbarrier, and warp 0
// refills the slot once all have; no CTA-wide barrier runs in the loop, so
// warps may drift a stage apart.  Each CTA writes its unnormalised partial
// output with its running max and sum; a second kernel (launched as a
// programmatic dependent of the first) merges the partials by log-sum-exp,
// one CTA per (head, 32-channel slice).  With G = 1 every key is local and a separate
// instantiation without the remote path runs.
//
// The same kernels run a prefill chunk (§3.1, §3.2): n queries at positions
// P0 .. P0+n-1 are n problems over one cache (grid z = batch x query), each
// over keys [0, its position], with one G for the call; splits past a
// query's last key write empty partials, which the combine weighs by zero.
//
// Traffic: K and V once (2 * L * Hkv * D * 2 bytes per token of output);
// everything else is O(Hq * D * n_split).
#include <cmath>
#include <type_traits>

#include "jl_common.cuh"
#include "sm100_ptx.cuh"

namespace jl {
namespace {

constexpr int kDecWarps = 8;  // warps = KV heads per CTA
constexpr int kDecThreads = kDecWarps * 32;
constexpr int kStages = 3;
constexpr int kCtasPerSm = 2;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

template <int D>
struct DecCfg {
  static constexpr int P = D == 128 ? 8 : 16;   // tokens per stage
  static constexpr int NBLK = P / 8;            // 8-token score blocks per stage
  static constexpr int KB = D / 16;             // 16-channel k-blocks
  static constexpr int ROW = kDecWarps * D * 2 + 16;  // padded token row (all CTA heads)
  static constexpr int HALF_STAGE = P * ROW;          // K (or V) of a stage
  static constexpr int STAGE = 2 * HALF_STAGE;
  // cos/sin row of one token: (cos, sin) per frequency, padded so two rows
  // read in one 128 B wavefront use different banks (D = 128; at D = 64 the
  // full padding would not leave room for two CTAs per SM).
  static constexpr int CS_ROW = (D / 2) * 8 + (D == 128 ? 64 : 16);
  static constexpr int CS_TAB = P * CS_ROW;           // one stage's correction table
  static constexpr int CS = kStages * STAGE;          // kStages tables (one per slot)
  static constexpr int OMEGA = CS + kStages * CS_TAB;  // theta_i / (2 pi), 0.64 fixed point
  static constexpr int QCS = OMEGA + (D / 2) * 8;      // (cos, sin) at p and f(p), [2][D/2]
  static constexpr int BAR = QCS + 2 * (D / 2) * 8;    // full, empty, tready [kStages] each
  static constexpr int ABORT = BAR + 24 * kStages + 8;
  static constexpr int BYTES = ABORT + 16;  // about 112 KB (D = 128): two CTAs per SM
};
static_assert(kCtasPerSm * (DecCfg<128>::BYTES + 1024) <= 233472, "two CTAs per SM");
static_assert(kCtasPerSm * (DecCfg<64>::BYTES + 1024) <= 233472, "two CTAs per SM");

__device__ __forceinline__ void bulk_copy(uint32_t dst, const void *src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

// D(16x8, f32) += A(16x16) * B(16x8) with FP16 or BF16 operands (register fragments).
__device__ __forceinline__ void mma_f16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                        uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Pack (lo, hi) as f16x2 / bf16x2 (lo in the low half = lower index).
__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
__device__ __forceinline__ float2 fmul2(float2 a, float2 b) {
  float2 d;
  asm("{.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
__device__ __forceinline__ float2 fsub2(float2 a, float2 b) {
  float2 d;
  asm("{.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "sub.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
__device__ __forceinline__ float bf_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf_hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }

// S (16 x 8, rows = the group's heads, columns = 8 tokens) += Q K^T over the
// k-blocks [kb0, kb0 + 2) and their RoPE partners [kb0 + KB/2, kb0 + KB/2 + 2).
// K is read with ldmatrix as FP16-converted B fragments; remote tokens are
// first turned by the correction rotation (channel c pairs with c + D/2).
// How a stage's key rows are turned into FP16 B fragments.
enum KeyKind : int {
  kKeyBf16 = 0,    // cached BF16 key at its true position: converted
  kKeyRotate = 1,  // cached BF16 key of a remote token: turned by R(Delta j), converted
  kKeyF16 = 2,     // remote form of the key, stored as FP16: used as read
};

template <int D, int KIND>
__device__ __forceinline__ void qk_pair(float (&sc)[4], const uint32_t (&q)[D / 16][2],
                                        uint32_t krow_addr, const uint8_t *cs_row, int kb0,
                                        int tq, int mat) {
  constexpr int HK = D / 32;  // k-block offset of the RoPE partners
  uint32_t lo[4], hi[4];      // k-blocks kb0, kb0 + 1 and their partners
  ldsm_x4(krow_addr + (16 * kb0 + 8 * (mat & 1) + 16 * (mat >> 1)) * 2, lo);
  ldsm_x4(krow_addr + (16 * (kb0 + HK) + 8 * (mat & 1) + 16 * (mat >> 1)) * 2, hi);
  // kKeyF16: the ldmatrix fragments are the FP16 operand already
#pragma unroll
  for (int r = 0; r < (KIND == kKeyF16 ? 0 : 4); ++r) {
    const float x0 = bf_lo(lo[r]), x1 = bf_hi(lo[r]);
    const float y0 = bf_lo(hi[r]), y1 = bf_hi(hi[r]);
    if constexpr (KIND == kKeyRotate) {
      // lo[r]: channels c, c + 1 with c = 16 (kb0 + r / 2) + 8 (r % 2) + 2 tq
      const int c = 16 * (kb0 + (r >> 1)) + 8 * (r & 1) + 2 * tq;
      const float4 cs = *reinterpret_cast<const float4 *>(cs_row + c * 8);  // cos c, c+1, sin c, c+1
      const float2 xx = make_float2(x0, x1), yy = make_float2(y0, y1);
      const float2 co = make_float2(cs.x, cs.y), si = make_float2(cs.z, cs.w);
      const float2 l2 = fsub2(fmul2(xx, co), fmul2(yy, si));  // x cos - y sin
      const float2 h2 = ffma2(yy, co, fmul2(xx, si));         // x sin + y cos
      lo[r] = pack_f16(l2.x, l2.y);
      hi[r] = pack_f16(h2.x, h2.y);
    } else {
      lo[r] = pack_f16(x0, x1);
      hi[r] = pack_f16(y0, y1);
    }
  }
  mma_f16(sc, q[kb0][0], 0u, q[kb0][1], 0u, lo[0], lo[1]);
  mma_f16(sc, q[kb0 + 1][0], 0u, q[kb0 + 1][1], 0u, lo[2], lo[3]);
  mma_f16(sc, q[kb0 + HK][0], 0u, q[kb0 + HK][1], 0u, hi[0], hi[1]);
  mma_f16(sc, q[kb0 + HK + 1][0], 0u, q[kb0 + HK + 1][1], 0u, hi[2], hi[3]);
}

template <int D, int KIND>
__device__ __forceinline__ void qk_block(float (&sc)[4], const uint32_t (&q)[D / 16][2],
                                         uint32_t krow_addr, const uint8_t *cs_row, int tq,
                                         int mat) {
  // one accumulator chain: the other warps' work covers the MMA latency, and
  // two interleaved chains (more registers live) measured slower
#pragma unroll
  for (int kb0 = 0; kb0 < D / 32; kb0 += 2)
    qk_pair<D, KIND>(sc, q, krow_addr, cs_row, kb0, tq, mat);
}

// Rows of the correction table of one stage: cos and sin of Delta j * theta_i
// for token row tt (j = jt + tt) and frequency i < D/2, Delta j = f(j) - j,
// stored per channel pair (i, i+1) as (cos_i, cos_i+1, sin_i, sin_i+1).
// The phase in turns is Delta j * omega_i modulo 1, with omega_i =
// theta_i / (2 pi) as a 64-bit binary fraction: the 64-bit product wraps
// exactly, its top 32 bits are the signed phase in units of 2^-32 turn, and
// the angle handed to the sine/cosine lies in [-pi, pi).  Warp w writes rows
// w, w + nw, ... of the stage.  Under the frequency-interpolation remote map
// the correction angle is j (theta'_i - theta_i): Delta j = j, and omega_i
// holds (theta'_i - theta_i) / (2 pi), a negative fraction in two's complement.
template <int D>
__device__ __forceinline__ void correction_rows(uint8_t *tab, int jt, int n,
                                                const GroupDivider &gdiv, int interp, int warp,
                                                int nw, int lane, const uint64_t *omega) {
  using C = DecCfg<D>;
  constexpr float kTurnToRad = 1.4629180792671596e-09f;  // 2 pi / 2^32
  for (int tt = warp; tt < n; tt += nw) {
    const int j = jt + tt;
    const uint64_t delta =
        static_cast<uint64_t>(static_cast<int64_t>(interp ? j : remap_fast(j, gdiv) - j));
    if (lane < D / 4) {  // lane: channels 2 lane, 2 lane + 1
      const int i = 2 * lane;
      const int32_t p0 = static_cast<int32_t>((delta * omega[i]) >> 32);
      const int32_t p1 = static_cast<int32_t>((delta * omega[i + 1]) >> 32);
      float c0, s0, c1, s1;
      __sincosf(static_cast<float>(p0) * kTurnToRad, &s0, &c0);
      __sincosf(static_cast<float>(p1) * kTurnToRad, &s1, &c1);
      *reinterpret_cast<float4 *>(tab + tt * C::CS_ROW + i * 8) = make_float4(c0, c1, s0, s1);
    }
  }
}

// Bounded mbarrier wait that also gives up once another warp raised `abort`.
__device__ __forceinline__ bool dec_wait(uint32_t bar, uint32_t parity, volatile uint32_t *abort) {
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

// BIFOCAL = false is the G = 1 instantiation: every key is local, so it has
// no remote query, no correction table and no rotation code.  TWO_FORM (with
// BIFOCAL) reads remote tokens' keys from the FP16 remote form of the cache
// (a.k_remote, already turned by R(Delta j)) instead of rotating them: no
// correction table either.
template <int D, int GRP, bool BIFOCAL, bool TWO_FORM = false>
__global__ void __launch_bounds__(kDecThreads, kCtasPerSm)
decode_split_kernel(const __grid_constant__ DecodeArgs a) {
  using C = DecCfg<D>;
  constexpr int P = C::P, NBLK = C::NBLK, KB = C::KB, HALF = D / 2, MB = D / 16;

  extern __shared__ __align__(128) uint8_t dsm[];
  const uint32_t sb = smem_u32(dsm);
  volatile uint32_t *abort = reinterpret_cast<volatile uint32_t *>(dsm + C::ABORT);
  auto full = [&](int slot) { return sb + C::BAR + 8u * static_cast<uint32_t>(slot); };
  auto empty = [&](int slot) { return sb + C::BAR + 8u * static_cast<uint32_t>(kStages + slot); };
  auto tready = [&](int slot) { return sb + C::BAR + 8u * static_cast<uint32_t>(2 * kStages + slot); };

  const int s = blockIdx.x, chunk_id = blockIdx.y, bq = blockIdx.z;  // bq = b * nq + query
  const int b = bq / a.nq;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g0 = chunk_id * kDecWarps;
  const int nh = min(kDecWarps, a.Hkv - g0);  // KV heads of this CTA = working warps
  const int p = a.q_pos0 + (bq - b * a.nq);  // this query's position; keys [0, p]
  const int w0eff = BIFOCAL ? a.w0 : INT_MAX;
  const int j_begin = s * a.chunk;
  const int j_end = min(p + 1, j_begin + a.chunk);  // may be <= j_begin: an empty split
  const int n_stage = (j_end - j_begin + P - 1) / P;
  const uint32_t head_bytes = static_cast<uint32_t>(nh) * D * 2;  // one token, CTA heads
  const size_t cache_row = static_cast<size_t>(a.Hkv) * D;        // elements per token

  // RoPE frequencies as turns per position and the query's cos/sin at p and
  // f(p), once per CTA.
  uint64_t *omega = reinterpret_cast<uint64_t *>(dsm + C::OMEGA);
  float2 *qcs = reinterpret_cast<float2 *>(dsm + C::QCS);
  int n_issued = 0;  // warp 0: stages whose copies are posted
  // One bulk copy per token and tensor into rows padded by 16 B (bank-conflict
  // free ldmatrix), posted by warp 0: lane 0 adds the byte count, lanes
  // [0, 2P) each issue one copy.  Slots past the chunk end repeat its last
  // token, so every row the tensor core reads holds finite data; those tokens
  // are masked.
  auto issue = [&](int u) {  // warp 0, all lanes
    ++n_issued;
    const int slot = u % kStages;
    const int ju = j_begin + u * P;
    if (lane == 0) mbar_arrive_expect_tx(full(slot), 2u * P * head_bytes);
    __syncwarp();
    if (lane < 2 * P) {
      const int t2 = lane >> 1;
      const int j = min(ju + t2, j_end - 1);
      const size_t off = (static_cast<size_t>(b) * a.Lcap + j) * cache_row + static_cast<size_t>(g0) * D;
      const uint32_t dst = sb + slot * C::STAGE + (lane & 1) * C::HALF_STAGE + t2 * C::ROW;
      const void *src = (lane & 1) ? static_cast<const void *>(a.v_cache + off)
                        : (TWO_FORM && p - j > w0eff) ? static_cast<const void *>(a.k_remote + off)
                                                      : static_cast<const void *>(a.k_cache + off);
      bulk_copy(dst, src, head_bytes, full(slot));
    }
  };
  // This warp's rows of the correction table of stage u (table u % kStages),
  // then its arrival on that table's barrier; the table's previous user,
  // stage u - kStages, must be done in every warp first.
  auto table = [&](int u) -> bool {
    if (u >= kStages) {
      const bool got = dec_wait(empty(u % kStages), static_cast<uint32_t>(u / kStages - 1) & 1u, abort);
      if (!__all_sync(0xffffffffu, got)) return false;
    }
    const int ju = j_begin + u * P;
    if (p - ju > w0eff)
      correction_rows<D>(dsm + C::CS + (u % kStages) * C::CS_TAB, ju, min(P, j_end - ju), a.gdiv,
                         a.interp, warp, nh, lane, omega);
    __syncwarp();
    if (lane == 0) mbar_arrive(tready(u % kStages));
    return true;
  };
  if (warp == 0) {
    if (lane == 0) {
      for (int i = 0; i < kStages; ++i) {
        mbar_init(full(i), 1);    // copies posted, completes when their bytes land
        mbar_init(empty(i), nh);  // one arrival per working warp
      }
      for (int i = 0; i < kStages; ++i) mbar_init(tready(i), nh);  // table rows written
      *abort = 0u;
      fence_mbar_init();
    }
    __syncwarp();
    // The first copies go out before the RoPE tables are computed.
    for (int u = 0; u < kStages && u < n_stage; ++u) issue(u);
  }
  // The turn fractions per position come with the call (formed once on the
  // host); the query's angles are exact modulo one turn like the table's.
  constexpr float kTurnToRad = 1.4629180792671596e-09f;  // 2 pi / 2^32
  for (int i = tid; i < HALF; i += kDecThreads) omega[i] = a.omega_corr[i];
  const uint64_t pos_r = static_cast<uint64_t>(a.interp ? p : remap_fast(p, a.gdiv));
  for (int idx = tid; idx < 2 * HALF; idx += kDecThreads) {
    const int i = idx < HALF ? idx : idx - HALF;
    // RoPE(x_q, p), and the remote query: RoPE(x_q, f(p)), or RoPE'(x_q, p)
    // (true position, interpolated frequency)
    const uint64_t turns = idx < HALF ? static_cast<uint64_t>(p) * a.omega_qt[i]
                                      : pos_r * a.omega_qr[i];
    float c, sn;
    __sincosf(static_cast<float>(static_cast<int32_t>(turns >> 32)) * kTurnToRad, &sn, &c);
    qcs[idx] = make_float2(c, sn);
  }
  __syncthreads();
  if (warp >= nh) return;  // no KV head for this warp; nothing below waits for it
  bool ok = true;
  if constexpr (BIFOCAL && !TWO_FORM) {
    ok = table(0);
    if (ok && n_stage > 1) ok = table(1);
  }

  // Query fragments (A operand, rows = the group's heads, FP16, pre-scaled by
  // log2(e)/sqrt(D)) at the true position p and the remote position f(p).
  // Row gq holds query head gq of the group; rows >= GRP (and 8..15) are zero.
  const int gq = lane >> 2, tq = lane & 3;     // mma fragment coordinates
  const int mat = lane >> 3, mrow = lane & 7;  // ldmatrix: matrix and row this lane addresses
  const int g = g0 + warp;
  const float qscale = kLog2e / sqrtf(static_cast<float>(D));
  uint32_t qt[KB][2], qr[KB][2];
  {
    const bool qrow_ok = gq < GRP;
    const __nv_bfloat16 *qrow = a.q + (static_cast<size_t>(bq) * a.Hq + g * GRP + (qrow_ok ? gq : 0)) * D;
#pragma unroll
    for (int kb = 0; kb < KB / 2; ++kb)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float vt[2][2], vr[2][2];  // [first / partner][channel c0, c0 + 1]
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int c = 16 * kb + 2 * tq + 8 * h + e;  // first member, < D/2
          const float x = qrow_ok ? bf2f(qrow[c]) : 0.f;
          const float y = qrow_ok ? bf2f(qrow[c + HALF]) : 0.f;
          const float2 ct = qcs[c], cr = qcs[HALF + c];
          vt[0][e] = (x * ct.x - y * ct.y) * qscale;
          vt[1][e] = (x * ct.y + y * ct.x) * qscale;
          vr[0][e] = (x * cr.x - y * cr.y) * qscale;
          vr[1][e] = (x * cr.y + y * cr.x) * qscale;
        }
        qt[kb][h] = pack_f16(vt[0][0], vt[0][1]);
        qt[kb + KB / 2][h] = pack_f16(vt[1][0], vt[1][1]);
        qr[kb][h] = pack_f16(vr[0][0], vr[0][1]);
        qr[kb + KB / 2][h] = pack_f16(vr[1][0], vr[1][1]);
      }
  }

  // O^T accumulators: m-block mb holds (channel 16mb + gq, heads 2tq, 2tq+1)
  // in o[mb][0..1] and channel 16mb + gq + 8 in o[mb][2..3].
  float o[MB][4];
#pragma unroll
  for (int mb = 0; mb < MB; ++mb)
#pragma unroll
    for (int e = 0; e < 4; ++e) o[mb][e] = 0.f;
  float m_run = -INFINITY;  // running max (base 2) of head gq, same in its 4 lanes
  float l_part = 0.f;       // this lane's share of head gq's running sum
  const uint32_t warp_col = static_cast<uint32_t>(warp) * D * 2;

  int slot = 0;
  uint32_t phase = 0;
  // The stage loop, in two copies: CTAs whose whole chunk lies beyond the
  // local window (all but the last few splits) run one without the local and
  // window-edge paths, which needs fewer live registers.
  auto stage_loop = [&](auto remote_only_tag) {
  constexpr bool RO = decltype(remote_only_tag)::value;
  for (int t = 0; t < n_stage && ok; ++t) {
    const int jt = j_begin + t * P;
    const int n = min(P, j_end - jt);
    ok = dec_wait(full(slot), phase, abort) &&
         (!BIFOCAL || TWO_FORM || dec_wait(tready(slot), phase, abort));
    if (!__all_sync(0xffffffffu, ok)) {
      ok = false;
      break;
    }
    {
      const uint32_t kst = sb + slot * C::STAGE + warp_col;
      const uint32_t vst = kst + C::HALF_STAGE;
      const uint8_t *tab = dsm + C::CS + slot * C::CS_TAB;
      // Scores of head gq for tokens tb + 2tq, tb + 2tq + 1 of each 8-token
      // block; every block of the stage is scored before the running max
      // moves, since one P.V product covers all of them.
      float sv[NBLK][2];
#pragma unroll
      for (int nb = 0; nb < NBLK; ++nb) {
        const int tb = nb * 8;
        const uint32_t krow = kst + (tb + mrow) * C::ROW;
        const uint8_t *cs_row = tab + (tb + gq) * C::CS_ROW;  // this lane's token gq
        const int jb = jt + tb;
        const int nb_valid = min(8, n - tb);
        const bool all_remote = p - (jb + 7) > w0eff;
        const bool all_local = p - jb <= w0eff;
        float sc[4] = {0.f, 0.f, 0.f, 0.f};
        constexpr int kRemoteKind = TWO_FORM ? kKeyF16 : kKeyRotate;
        if (!BIFOCAL) {
          qk_block<D, kKeyBf16>(sc, qt, krow, cs_row, tq, mat);
        } else if (RO || all_remote) {
          qk_block<D, kRemoteKind>(sc, qr, krow, cs_row, tq, mat);
        } else if (all_local) {
          qk_block<D, kKeyBf16>(sc, qt, krow, cs_row, tq, mat);
        } else {  // the block on the window edge: both variants, picked per token
          // (with TWO_FORM the rows of one variant hold the other's format;
          // those columns of S are computed but never picked)
          float sl[4] = {0.f, 0.f, 0.f, 0.f};
          qk_block<D, kRemoteKind>(sc, qr, krow, cs_row, tq, mat);
          qk_block<D, kKeyBf16>(sl, qt, krow, cs_row, tq, mat);
          if (p - (jb + 2 * tq) <= w0eff) sc[0] = sl[0];
          if (p - (jb + 2 * tq + 1) <= w0eff) sc[1] = sl[1];
        }
        sv[nb][0] = 2 * tq < nb_valid ? sc[0] : -INFINITY;
        sv[nb][1] = 2 * tq + 1 < nb_valid ? sc[1] : -INFINITY;
      }
      float bm = fmaxf(sv[0][0], sv[0][1]);
#pragma unroll
      for (int nb = 1; nb < NBLK; ++nb) bm = fmaxf(bm, fmaxf(sv[nb][0], sv[nb][1]));
      bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 1));
      bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 2));
      // lazy online softmax: the reference max moves only when it grows by
      // more than 2^8 (O and l share it, so the result is exact)
      float alpha = 1.f;
      if (bm > m_run + kRescaleThreshold || (m_run == -INFINITY && bm > -INFINITY)) {
        if (m_run != -INFINITY) alpha = exp2f(m_run - bm);
        m_run = bm;
      }
      if (__any_sync(0xffffffffu, alpha != 1.f)) {
        // O^T columns are heads 2tq, 2tq+1; their factors live in lanes 4*head
        const float a0 = __shfl_sync(0xffffffffu, alpha, (2 * tq) * 4);
        const float a1 = __shfl_sync(0xffffffffu, alpha, (2 * tq + 1) * 4);
#pragma unroll
        for (int mb = 0; mb < MB; ++mb) {
          o[mb][0] *= a0;
          o[mb][1] *= a1;
          o[mb][2] *= a0;
          o[mb][3] *= a1;
        }
        l_part *= alpha;
      }
      const float neg_m = m_run == -INFINITY ? 0.f : -m_run;
      uint32_t pfrag[NBLK];  // P^T fragments (BF16), one per 8-token block
#pragma unroll
      for (int nb = 0; nb < NBLK; ++nb) {
        const float p0 = ex2_sfu(sv[nb][0] + neg_m), p1 = ex2_sfu(sv[nb][1] + neg_m);
        l_part += p0 + p1;
        pfrag[nb] = pack_bf16(p0, p1);
      }
      // O^T += V^T P^T over this stage's tokens (k = 16 tokens; with 8-token
      // stages the upper half of P is zero and V's rows are reused)
      const uint32_t pb0 = pfrag[0], pb1 = NBLK > 1 ? pfrag[NBLK - 1] : 0u;
#pragma unroll
      for (int mb = 0; mb < MB; mb += 2) {
        uint32_t lo[4];
        ldsm_x4_t(vst + mrow * C::ROW + (16 * mb + 8 * (mat & 1) + 16 * (mat >> 1)) * 2, lo);
        if constexpr (NBLK > 1) {
          uint32_t hi[4];
          ldsm_x4_t(vst + (8 + mrow) * C::ROW + (16 * mb + 8 * (mat & 1) + 16 * (mat >> 1)) * 2, hi);
          mma_bf16(o[mb], lo[0], lo[1], hi[0], hi[1], pb0, pb1);
          mma_bf16(o[mb + 1], lo[2], lo[3], hi[2], hi[3], pb0, pb1);
        } else {
          mma_bf16(o[mb], lo[0], lo[1], lo[0], lo[1], pb0, pb1);
          mma_bf16(o[mb + 1], lo[2], lo[3], lo[2], lo[3], pb0, pb1);
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(empty(slot));
    // This warp's rows of the table two stages ahead.
    if (BIFOCAL && !TWO_FORM && t + 2 < n_stage) ok = table(t + 2);
    // Warp 0 refills this slot once every warp has released it.
    if (warp == 0 && ok && t + kStages < n_stage) {
      ok = __all_sync(0xffffffffu, dec_wait(empty(slot), phase, abort));
      if (ok) issue(t + kStages);
    }
    if (++slot == kStages) {
      slot = 0;
      phase ^= 1u;
    }
  }
  };
  if (BIFOCAL && p - (j_end - 1) > w0eff)
    stage_loop(std::true_type{});
  else
    stage_loop(std::false_type{});
  if (!ok || *abort) {
    // This warp stops.  Warp 0 first lets the copies it posted land
    // (bounded), so none writes into shared memory after the CTA exits: only
    // the last kStages stages it issued can be in flight, since a slot is
    // refilled only after every warp consumed its previous stage.
    if (lane == 0) {
      *abort = 1u;
      atomicOr(a.dev_error, kDevTimeout);
    }
    if (warp == 0 && lane == 0)
      for (int u = max(0, n_issued - kStages); u < n_issued; ++u)
        mbar_wait_bounded(full(u % kStages), static_cast<uint32_t>(u / kStages) & 1u, 2000000ull);
    return;
  }
  // Row sums: the four lanes of head gq hold its shares.
  float l_run = l_part + __shfl_xor_sync(0xffffffffu, l_part, 1);
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);
  // Partial record per query head: [D] unnormalised output, then the running
  // max (base 2) and sum.
  const size_t rec_stride = static_cast<size_t>(a.n_split) * (D + 2);
  float *rec0 = a.partial + ((static_cast<size_t>(bq) * a.Hq + g * GRP) * a.n_split + s) * (D + 2);
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const int h = 2 * tq + e;  // O^T column = query head of the group
    if (h < GRP) {
      float *rec = rec0 + h * rec_stride;
#pragma unroll
      for (int mb = 0; mb < MB; ++mb) {
        rec[16 * mb + gq] = o[mb][e];
        rec[16 * mb + gq + 8] = o[mb][2 + e];
      }
    }
  }
  if (tq == 0 && gq < GRP) {
    float *rec = rec0 + gq * rec_stride;
    rec[D] = m_run;
    rec[D + 1] = l_run;
  }
}

// Remote form of the key cache, for the two-form decode: for tokens
// j in [j0, j1) of batch entry blockIdx.y and every KV head,
//   k_remote[b, j, g, :] = FP16(R(f(j) - j) k_cache[b, j, g, :]),
// with G from the length L the cache will be read at.  The table rows come
// from correction_rows and the rotation is the packed sequence of qk_pair,
// so the decode kernel's tensor-core operands are the same either way.
// One warp per token, eight tokens per CTA; lane l turns channel pair
// (2l, 2l + 1) and its RoPE partners.
template <int D>
__global__ void __launch_bounds__(kDecThreads)
remote_cache_kernel(const __nv_bfloat16 *__restrict__ k_cache, __half *__restrict__ k_remote,
                    int Lcap, int Hkv, int j0, int j1, GroupDivider gdiv, float theta) {
  using C = DecCfg<D>;
  constexpr int HALF = D / 2;
  __shared__ __align__(16) uint8_t tab[kDecWarps * C::CS_ROW];
  __shared__ uint64_t omega[HALF];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.y;
  const int jt = j0 + blockIdx.x * kDecWarps;
  const int n = min(kDecWarps, j1 - jt);
  constexpr double kTurnsQ64 = 0.15915494309189533577 * 18446744073709551616.0;  // 2^64 / (2 pi)
  for (int i = threadIdx.x; i < HALF; i += kDecThreads)
    omega[i] = __double2ull_rn(rope_freq(i, D, static_cast<double>(theta)) * kTurnsQ64);
  __syncthreads();
  correction_rows<D>(tab, jt, n, gdiv, 0, warp, kDecWarps, lane, omega);  // row `warp`
  __syncwarp();
  if (warp >= n || lane >= D / 4) return;
  const int c = 2 * lane;
  const float4 cs = *reinterpret_cast<const float4 *>(tab + warp * C::CS_ROW + c * 8);
  const float2 co = make_float2(cs.x, cs.y), si = make_float2(cs.z, cs.w);
  const size_t row0 = (static_cast<size_t>(b) * Lcap + jt + warp) * Hkv * D;
  for (int g = 0; g < Hkv; ++g) {
    const size_t row = row0 + static_cast<size_t>(g) * D;
    const uint32_t lo = *reinterpret_cast<const uint32_t *>(k_cache + row + c);
    const uint32_t hi = *reinterpret_cast<const uint32_t *>(k_cache + row + c + HALF);
    const float2 xx = make_float2(bf_lo(lo), bf_hi(lo)), yy = make_float2(bf_lo(hi), bf_hi(hi));
    const float2 l2 = fsub2(fmul2(xx, co), fmul2(yy, si));  // x cos - y sin
    const float2 h2 = ffma2(yy, co, fmul2(xx, si));         // x sin + y cos
    *reinterpret_cast<uint32_t *>(k_remote + row + c) = pack_f16(l2.x, l2.y);
    *reinterpret_cast<uint32_t *>(k_remote + row + c + HALF) = pack_f16(h2.x, h2.y);
  }
}

// Merge the split partials of one (b, head) for one 32-channel slice, one
// CTA of 8 warps: the block-wide max of the split maxima and the weights
// 2^(m_s - M) (one round of loads), then warp w sums splits w, w + 8, ... for
// channel `lane` of the slice with every load issued up front (the loop is
// unrolled to the largest split count), and the 8 warp sums are added.
// Launched as a programmatic dependent of the split kernel: the wait below
// returns once that grid has finished and its partials are visible.
constexpr int kCombineThreads = 256;
constexpr int kCombineWarps = kCombineThreads / 32;
constexpr int kMaxSplit = kCtasPerSm * 148;  // decode_plan never exceeds this
constexpr int kSplitsPerWarp = (kMaxSplit + kCombineWarps - 1) / kCombineWarps;
static_assert(kMaxSplit <= 2 * kCombineThreads, "two splits per thread in the max pass");

template <int D>
__global__ void __launch_bounds__(kCombineThreads)
decode_combine_kernel(const __grid_constant__ DecodeArgs a) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  __shared__ float wsh[kMaxSplit];
  __shared__ float red[kCombineWarps][32];
  __shared__ float part[kCombineWarps];
  const int bh = blockIdx.x;     // (b * nq + query) * Hq + head
  const int c = blockIdx.y * 32 + (threadIdx.x & 31);  // channel of this lane
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int ns = a.n_split;
  const float *rec = a.partial + static_cast<size_t>(bh) * ns * (D + 2);

  // the split maxima and sums, two splits per thread at most
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  if (tid < ns) {
    m0 = rec[tid * (D + 2) + D];
    l0 = rec[tid * (D + 2) + D + 1];
  }
  if (tid + kCombineThreads < ns) {
    m1 = rec[(tid + kCombineThreads) * (D + 2) + D];
    l1 = rec[(tid + kCombineThreads) * (D + 2) + D + 1];
  }
  float m = fmaxf(m0, m1);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) part[warp] = m;
  __syncthreads();
  float M = part[0];
#pragma unroll
  for (int w = 1; w < kCombineWarps; ++w) M = fmaxf(M, part[w]);
  __syncthreads();  // part[] is reused below
  float l = 0.f;
  if (tid < ns) {
    const float w = exp2f(m0 - M);
    wsh[tid] = w;
    l = l0 * w;
  }
  if (tid + kCombineThreads < ns) {
    const float w = exp2f(m1 - M);
    wsh[tid + kCombineThreads] = w;
    l = fmaf(l1, w, l);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
  if (lane == 0) part[warp] = l;
  __syncthreads();
  float lsum = 0.f;
#pragma unroll
  for (int w = 0; w < kCombineWarps; ++w) lsum += part[w];

  float v[kSplitsPerWarp];
#pragma unroll
  for (int k = 0; k < kSplitsPerWarp; ++k) {
    const int sp = warp + kCombineWarps * k;
    v[k] = (sp < ns && c < D) ? rec[static_cast<size_t>(sp) * (D + 2) + c] : 0.f;
  }
  float acc = 0.f;
#pragma unroll
  for (int k = 0; k < kSplitsPerWarp; ++k) {
    const int sp = warp + kCombineWarps * k;
    if (sp < ns) acc = fmaf(wsh[sp], v[k], acc);
  }
  red[warp][lane] = acc;
  __syncthreads();
  if (tid < 32 && c < D) {
    float o = 0.f;
#pragma unroll
    for (int w = 0; w < kCombineWarps; ++w) o += red[w][tid];
    o /= lsum;
    const size_t idx = static_cast<size_t>(bh) * D + c;
    if (a.out_f32)
      reinterpret_cast<float *>(a.out)[idx] = o;
    else
      reinterpret_cast<__nv_bfloat16 *>(a.out)[idx] = __float2bfloat16_rn(o);
  }
  if (blockIdx.y == 0 && tid == 0 && a.lse) {  // lse is [B, Hq, nq]
    const int h = bh % a.Hq, bqi = bh / a.Hq;
    const int bb = bqi / a.nq, qi = bqi - bb * a.nq;
    a.lse[(static_cast<size_t>(bb) * a.Hq + h) * a.nq + qi] = (M + log2f(lsum)) * 0.69314718055994531f;
  }
}

template <int D, int GRP, bool BIFOCAL, bool TWO_FORM>
cudaError_t launch_split_v(const DecodeArgs &a, cudaStream_t stream) {
  const int smem = DecCfg<D>::BYTES;
  cudaError_t e = ensure_smem_limit<decode_split_kernel<D, GRP, BIFOCAL, TWO_FORM>>(smem);
  if (e != cudaSuccess) return e;
  const int n_chunk = (a.Hkv + kDecWarps - 1) / kDecWarps;
  decode_split_kernel<D, GRP, BIFOCAL, TWO_FORM>
      <<<dim3(a.n_split, n_chunk, a.B * a.nq), kDecThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

template <int D, int GRP>
cudaError_t launch_split(const DecodeArgs &a, cudaStream_t stream) {
  if (a.G == 1) return launch_split_v<D, GRP, false, false>(a, stream);
  return a.k_remote ? launch_split_v<D, GRP, true, true>(a, stream)
                    : launch_split_v<D, GRP, true, false>(a, stream);
}

template <int D>
cudaError_t launch_decode_d(const DecodeArgs &a, cudaStream_t stream) {
  cudaError_t e;
  switch (a.Hq / a.Hkv) {
    case 1: e = launch_split<D, 1>(a, stream); break;
    case 2: e = launch_split<D, 2>(a, stream); break;
    case 4: e = launch_split<D, 4>(a, stream); break;
    case 8: e = launch_split<D, 8>(a, stream); break;
    default: return cudaErrorInvalidValue;
  }
  if (e != cudaSuccess) return e;
  if (a.n_split > kMaxSplit) return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(a.B * a.nq * a.Hq), D / 32);
  cfg.blockDim = dim3(kCombineThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, decode_combine_kernel<D>, a);
}

}  // namespace

void decode_plan(int B, int Hkv, int L, int *n_split, int *chunk) {
  // Two CTAs per SM (each holds a 3-stage ring of about 108 KB) over the 148
  // SMs of a B200; chunks are whole stages (8 or 16 tokens).  The split count
  // fills at most one wave of CTAs (rounding up would start a second,
  // nearly empty wave: 64 units x 5 splits = 320 CTAs for 296 slots).  It is
  // non-decreasing in L, so workspace sized for the largest L of a
  // generation loop covers every step.
  const int units = B * ((Hkv + kDecWarps - 1) / kDecWarps);
  int ns = (kCtasPerSm * 148) / units;
  const int max_ns = (L + 15) / 16;
  if (ns > max_ns) ns = max_ns;
  if (ns < 1) ns = 1;
  int ch = (L + ns - 1) / ns;
  ch = (ch + 15) / 16 * 16;  // a whole number of stages for both head dims
  *chunk = ch;
  *n_split = (L + ch - 1) / ch;
}

bool decode_supports_group(int grp) { return grp == 1 || grp == 2 || grp == 4 || grp == 8; }

cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t stream) {
  if (a.D == 128) return launch_decode_d<128>(a, stream);
  return launch_decode_d<64>(a, stream);
}

cudaError_t launch_split_merge(const float *partial, int n_split, void *out, int out_f32,
                               float *lse, int B, int nq, int Hq, int D, cudaStream_t stream) {
  if (n_split < 1 || n_split > kMaxSplit) return cudaErrorInvalidValue;
  DecodeArgs a{};
  a.partial = const_cast<float *>(partial);
  a.n_split = n_split;
  a.out = out;
  a.out_f32 = out_f32;
  a.lse = lse;
  a.B = B;
  a.nq = nq;
  a.Hq = Hq;
  a.D = D;
  // a plain launch: the dependency wait at the top of the merge returns at once
  const dim3 grid(static_cast<unsigned>(B * nq * Hq), D / 32);
  if (D == 128)
    decode_combine_kernel<128><<<grid, kCombineThreads, 0, stream>>>(a);
  else
    decode_combine_kernel<64><<<grid, kCombineThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_remote_cache(const __nv_bfloat16 *k_cache, __half *k_remote, int B, int Lcap,
                                int Hkv, int D, int j0, int j1, int G, float theta,
                                cudaStream_t stream) {
  const dim3 grid((j1 - j0 + kDecWarps - 1) / kDecWarps, B);
  if (D == 128)
    remote_cache_kernel<128><<<grid, kDecThreads, 0, stream>>>(k_cache, k_remote, Lcap, Hkv, j0,
                                                                j1, make_group_divider(G), theta);
  else
    remote_cache_kernel<64><<<grid, kDecThreads, 0, stream>>>(k_cache, k_remote, Lcap, Hkv, j0,
                                                               j1, make_group_divider(G), theta);
  return cudaGetLastError();
}

}  // namespace jl
