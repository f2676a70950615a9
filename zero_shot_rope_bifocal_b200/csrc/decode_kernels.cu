// decode_kernels.cu -- one generation step of bifocal attention on the
// true-position KV cache (Jet-Long paper, §3.2 "Key-value cache management and
// correction rotation"; score rule of §3; schedule of §3.1 with L = tokens in
// the cache including the new one, query at p = L - 1).
//
// Split-KV: CTA (s, c, b) streams key chunk s of KV heads [8c, 8c + 8) of
// batch b through a three-stage shared-memory ring filled by bulk async copies
// (cp.async.bulk + mbarrier transaction counts): each stage holds P tokens of
// K and V for the CTA's heads, which are contiguous in the cache.  Two CTAs
// share an SM, so 16 warps hide each other's shuffle and shared-memory
// latencies.  Warp w owns
// KV head 8c + w and its Hq/Hkv query heads; lane l holds channel pairs
// (i, i + D/2) for i in {2l, 2l+1} (D = 128) or {l} (D = 64), so the
// correction rotation of a pair is lane-local.
//
// Per token j: keys with p - j <= w0 are scored as cached against
// RoPE(x_q, p); older keys are first rotated by Delta j = f(j) - j (the
// correction rotation, so the cache is never rewritten) and scored against
// RoPE(x_q, f(p)).  cos/sin of Delta j * theta_i are evaluated once per token
// per CTA (double-precision angle, reduced, then the hardware sine/cosine on
// [-pi, pi]) and shared by all heads.  The partial dot products of a batch of
// tokens x query heads (32 values per lane) are summed across the warp by a
// reduce-scatter that leaves one (token, head) score per lane; an online
// softmax per head then weights V.  Each CTA writes its unnormalised partial
// output with its running max and sum; a second kernel merges the partials by
// log-sum-exp, one warp per head.
//
// Traffic: K and V once (2 * L * Hkv * D * 2 bytes per token of output);
// everything else is O(Hq * D * n_split).
#include <cmath>

#include "jl_common.cuh"
#include "sm100_ptx.cuh"

namespace jl {
namespace {

constexpr int kDecWarps = 8;  // = KV heads per CTA
constexpr int kDecThreads = kDecWarps * 32;
constexpr int kStages = 3;
constexpr int kCtasPerSm = 2;
constexpr float kLog2e = 1.4426950408889634f;

template <int D>
struct DecCfg {
  static constexpr int P = D == 128 ? 8 : 16;      // tokens per stage
  static constexpr int EPL = D / 32;               // channels per lane
  static constexpr int HEAD_BYTES = D * 2;         // one head's K (or V) row
  static constexpr int STAGE_HALF = P * kDecWarps * HEAD_BYTES;  // K (or V) of a stage: 16 KB
  static constexpr int STAGE = 2 * STAGE_HALF;
  static constexpr int CS = kStages * STAGE;                     // cos/sin table [P][D/2]
  static constexpr int BAR = CS + P * (D / 2) * 8;
  static constexpr int BYTES = BAR + 8 * kStages + 16;  // about 100 KB: two CTAs per SM
};

// Channel held by slot e of lane l: slots [0, EPL/2) are the first members of
// the lane's channel pairs, slots [EPL/2, EPL) their partners (+ D/2).
template <int D>
__device__ __forceinline__ int chan(int l, int e) {
  if constexpr (D == 128) return (e & 1) + 2 * l + (e >> 1) * 64;  // 2l, 2l+1, 64+2l, 65+2l
  else return l + e * 32;                                          // l, 32+l
}

// The lane's EPL channels of one BF16 head row in shared memory, as fp32.
template <int D>
__device__ __forceinline__ void load_row(const __nv_bfloat16 *row, int lane, float (&x)[D / 32]) {
  if constexpr (D == 128) {
    const __nv_bfloat162 lo = *reinterpret_cast<const __nv_bfloat162 *>(row + 2 * lane);
    const __nv_bfloat162 hi = *reinterpret_cast<const __nv_bfloat162 *>(row + 64 + 2 * lane);
    x[0] = __low2float(lo);
    x[1] = __high2float(lo);
    x[2] = __low2float(hi);
    x[3] = __high2float(hi);
  } else {
    x[0] = bf2f(row[lane]);
    x[1] = bf2f(row[lane + 32]);
  }
}

__device__ __forceinline__ void bulk_copy(uint32_t dst, const void *src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

// Sum NV per-lane values (v[0..NV)) across the warp.  Halving steps whose
// offset is at least NV add whole arrays; the remaining steps scatter, so that
// lane l ends with the warp total of value (l % NV).
template <int NV>
__device__ __forceinline__ float reduce_scatter(float (&v)[32], int lane) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    if (o >= NV) {
#pragma unroll
      for (int k = 0; k < NV; ++k) v[k] += __shfl_xor_sync(0xffffffffu, v[k], o);
    } else {
      const bool up = lane & o;
#pragma unroll
      for (int k = 0; k < o; ++k) {
        const float send = up ? v[k] : v[k + o];
        const float keep = up ? v[k + o] : v[k];
        v[k] = keep + __shfl_xor_sync(0xffffffffu, send, o);
      }
    }
  }
  return v[0];
}

// Partial dot products of one cached key (the lane's channels) with the
// group's queries; remote keys are first turned by the correction rotation.
template <int D, int GRP, bool REMOTE>
__device__ __forceinline__ void token_partials(float (&part)[32], int slot0,
                                               const __nv_bfloat16 *krow, const float2 *cs_row,
                                               int lane, const float (&q)[GRP][D / 32]) {
  constexpr int EPL = D / 32;
  float kv[EPL];
  load_row<D>(krow, lane, kv);
  if constexpr (REMOTE) {
    float2 cs[EPL / 2];
    if constexpr (D == 128) {
      const float4 c4 = *reinterpret_cast<const float4 *>(cs_row + 2 * lane);
      cs[0] = make_float2(c4.x, c4.y);
      cs[1] = make_float2(c4.z, c4.w);
    } else {
      cs[0] = cs_row[lane];
    }
#pragma unroll
    for (int e = 0; e < EPL / 2; ++e) {
      const float x = kv[e], y = kv[e + EPL / 2];
      kv[e] = x * cs[e].x - y * cs[e].y;
      kv[e + EPL / 2] = x * cs[e].y + y * cs[e].x;
    }
  }
#pragma unroll
  for (int h = 0; h < GRP; ++h) {
    float d = q[h][0] * kv[0];
#pragma unroll
    for (int e = 1; e < EPL; ++e) d = fmaf(q[h][e], kv[e], d);
    part[slot0 + h] = d;
  }
}

template <int D, int GRP>
__global__ void __launch_bounds__(kDecThreads, kCtasPerSm)
decode_split_kernel(DecodeArgs a) {
  using C = DecCfg<D>;
  constexpr int P = C::P, EPL = C::EPL, HALF = D / 2;
  constexpr int NB = (32 / GRP) < P ? (32 / GRP) : P;  // tokens per score batch
  constexpr int NV = NB * GRP;                         // values per batch: 8, 16 or 32
  static_assert(NV == 8 || NV == 16 || NV == 32, "batch must fill 8, 16 or 32 values");
  static_assert(P % NB == 0, "batches tile a stage");

  extern __shared__ __align__(128) uint8_t dsm[];
  const uint32_t sb = smem_u32(dsm);
  float2 *cs_tab = reinterpret_cast<float2 *>(dsm + C::CS);  // [P][D/2] (cos, sin)

  const int s = blockIdx.x, chunk_id = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g0 = chunk_id * kDecWarps;
  const int nh = min(kDecWarps, a.Hkv - g0);  // KV heads of this CTA
  const int g = g0 + warp;
  const bool wactive = warp < nh;
  const int p = a.L - 1;
  const int G = a.G;
  const int w0eff = (G == 1) ? INT_MAX : a.w0;
  const int j_begin = s * a.chunk;
  const int j_end = min(a.L, j_begin + a.chunk);
  const int n_stage = (j_end - j_begin + P - 1) / P;
  const uint32_t row_bytes = static_cast<uint32_t>(nh) * C::HEAD_BYTES;  // one token, CTA heads
  const size_t cache_row = static_cast<size_t>(a.Hkv) * D;               // elements per token

  if (tid == 0) {
    for (int i = 0; i < kStages; ++i) mbar_init(sb + C::BAR + 8 * i, 1);
    fence_mbar_init();
  }
  __syncthreads();

  auto issue = [&](int t) {
    const int slot = t % kStages;
    const int jt = j_begin + t * P;
    const int n = min(P, j_end - jt);
    const uint32_t bar = sb + C::BAR + 8 * slot;
    const uint32_t kdst = sb + slot * C::STAGE, vdst = kdst + C::STAGE_HALF;
    mbar_arrive_expect_tx(bar, 2u * n * row_bytes);
    const __nv_bfloat16 *ks = a.k_cache + (static_cast<size_t>(b) * a.Lcap + jt) * cache_row + g0 * D;
    const __nv_bfloat16 *vs = a.v_cache + (static_cast<size_t>(b) * a.Lcap + jt) * cache_row + g0 * D;
    if (nh == a.Hkv) {  // the CTA's rows of consecutive tokens are contiguous
      bulk_copy(kdst, ks, n * row_bytes, bar);
      bulk_copy(vdst, vs, n * row_bytes, bar);
    } else {
      for (int t2 = 0; t2 < n; ++t2) {
        bulk_copy(kdst + t2 * row_bytes, ks + t2 * cache_row, row_bytes, bar);
        bulk_copy(vdst + t2 * row_bytes, vs + t2 * cache_row, row_bytes, bar);
      }
    }
  };
  if (tid == 0)
    for (int t = 0; t < kStages && t < n_stage; ++t) issue(t);

  // Queries of this warp's heads at the true position p and the remote
  // position f(p), for the lane's channels, pre-scaled by log2(e)/sqrt(D).
  const double theta = static_cast<double>(a.theta);
  const float qscale = kLog2e / sqrtf(static_cast<float>(D));
  float qt[GRP][EPL], qr[GRP][EPL];
  {
    float ct[EPL / 2], st[EPL / 2], cr[EPL / 2], sr[EPL / 2];
#pragma unroll
    for (int e = 0; e < EPL / 2; ++e) {
      const double fr = rope_freq(chan<D>(lane, e), D, theta);
      rope_cos_sin(p, fr, ct[e], st[e]);
      rope_cos_sin(remap(p, G), fr, cr[e], sr[e]);
    }
#pragma unroll
    for (int h = 0; h < GRP; ++h) {
      const int hq = (wactive ? g : g0) * GRP + h;
      const __nv_bfloat16 *qrow = a.q + (static_cast<size_t>(b) * a.Hq + hq) * D;
#pragma unroll
      for (int e = 0; e < EPL / 2; ++e) {
        const float x = bf2f(qrow[chan<D>(lane, e)]), y = bf2f(qrow[chan<D>(lane, e) + HALF]);
        qt[h][e] = (x * ct[e] - y * st[e]) * qscale;
        qt[h][e + EPL / 2] = (x * st[e] + y * ct[e]) * qscale;
        qr[h][e] = (x * cr[e] - y * sr[e]) * qscale;
        qr[h][e + EPL / 2] = (x * sr[e] + y * cr[e]) * qscale;
      }
    }
  }

  float acc[GRP][EPL];
#pragma unroll
  for (int h = 0; h < GRP; ++h)
#pragma unroll
    for (int e = 0; e < EPL; ++e) acc[h][e] = 0.f;
  float m_mine = -INFINITY, l_mine = 0.f;  // state of head (lane % GRP)

  bool ok = true;
  int t_fail = 0;
  for (int t = 0; t < n_stage; ++t) {
    const int slot = t % kStages;
    const int jt = j_begin + t * P;
    const int n = min(P, j_end - jt);
    // cos/sin of the correction angles of this stage's remote tokens
    if (p - jt > w0eff) {
      for (int idx = tid; idx < n * HALF; idx += kDecThreads) {
        const int tt = idx / HALF, i = idx - tt * HALF;
        const int j = jt + tt;
        float c = 1.f, sn = 0.f;
        if (p - j > w0eff) {
          const double ang = static_cast<double>(remap(j, G) - j) *
                             rope_freq(i, D, theta);  // Delta j * theta_i
          const double r = ang - rint(ang * 0.15915494309189533577) * 6.283185307179586232;
          __sincosf(static_cast<float>(r), &sn, &c);
        }
        cs_tab[tt * HALF + i] = make_float2(c, sn);
      }
    }
    const uint32_t bar = sb + C::BAR + 8 * slot;
    ok = mbar_wait_bounded(bar, static_cast<uint32_t>(t / kStages) & 1u, kWaitLimitNs);
    if (__syncthreads_or(!ok)) {
      ok = false;
      t_fail = t;
      break;
    }
    if (wactive) {
      const uint8_t *kst = dsm + slot * C::STAGE + warp * C::HEAD_BYTES;
      const uint8_t *vst = kst + C::STAGE_HALF;
#pragma unroll 1
      for (int tb = 0; tb < n; tb += NB) {
        // partial scores of NB tokens x GRP heads; the query variant is
        // chosen per batch (all remote / all local), per token only on the
        // batch that straddles the window edge
        float part[32];
#pragma unroll
        for (int k = 0; k < 32; ++k) part[k] = 0.f;
        const int nb = min(NB, n - tb);
        const int jb = jt + tb;
        const bool all_remote = p - (jb + nb - 1) > w0eff;
        const bool all_local = p - jb <= w0eff;
        auto krow = [&](int pb) {
          return reinterpret_cast<const __nv_bfloat16 *>(kst + (tb + pb) * row_bytes);
        };
        if (all_remote) {
#pragma unroll
          for (int pb = 0; pb < NB; ++pb)
            if (pb < nb)
              token_partials<D, GRP, true>(part, pb * GRP, krow(pb), cs_tab + (tb + pb) * HALF, lane, qr);
        } else if (all_local) {
#pragma unroll
          for (int pb = 0; pb < NB; ++pb)
            if (pb < nb)
              token_partials<D, GRP, false>(part, pb * GRP, krow(pb), cs_tab, lane, qt);
        } else {
#pragma unroll
          for (int pb = 0; pb < NB; ++pb)
            if (pb < nb) {
              if (p - (jb + pb) > w0eff)
                token_partials<D, GRP, true>(part, pb * GRP, krow(pb), cs_tab + (tb + pb) * HALF, lane, qr);
              else
                token_partials<D, GRP, false>(part, pb * GRP, krow(pb), cs_tab, lane, qt);
            }
        }
        const float sc = reduce_scatter<NV>(part, lane);
        const int my_pb = (lane % NV) / GRP;
        const float sv = my_pb < nb ? sc : -INFINITY;
        // online softmax for head (lane % GRP) over the batch
        float bm = sv;
#pragma unroll
        for (int o = GRP; o < NV; o <<= 1) bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, o));
        const float m_new = fmaxf(m_mine, bm);  // finite: the batch holds a valid token
        const float alpha_mine = exp2f(m_mine - m_new);
        const float pm = exp2f(sv - m_new);
        float ps = pm;
#pragma unroll
        for (int o = GRP; o < NV; o <<= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
        l_mine = l_mine * alpha_mine + ps;
        m_mine = m_new;
#pragma unroll
        for (int h = 0; h < GRP; ++h) {
          const float al = __shfl_sync(0xffffffffu, alpha_mine, h);
#pragma unroll
          for (int e = 0; e < EPL; ++e) acc[h][e] *= al;
        }
#pragma unroll
        for (int pb = 0; pb < NB; ++pb) {
          if (pb < nb) {
            float vv[EPL];
            load_row<D>(reinterpret_cast<const __nv_bfloat16 *>(vst + (tb + pb) * row_bytes), lane, vv);
#pragma unroll
            for (int h = 0; h < GRP; ++h) {
              const float pr = __shfl_sync(0xffffffffu, pm, pb * GRP + h);
#pragma unroll
              for (int e = 0; e < EPL; ++e) acc[h][e] = fmaf(pr, vv[e], acc[h][e]);
            }
          }
        }
      }
    }
    __syncthreads();  // stage slot and cos/sin table free again
    if (tid == 0 && t + kStages < n_stage) issue(t + kStages);
  }
  if (!ok) {
    // Stages t_fail .. t_fail + kStages - 1 may still be in flight: let them
    // land (bounded) before the CTA exits, then report.
    if (tid == 0) {
      for (int u = t_fail; u < n_stage && u < t_fail + kStages; ++u)
        mbar_wait_bounded(sb + C::BAR + 8 * (u % kStages), static_cast<uint32_t>(u / kStages) & 1u,
                          kWaitLimitNs);
      atomicOr(a.dev_error, kDevTimeout);
    }
    return;
  }
  if (!wactive) return;
  // Partial record: [D] unnormalised output, then the running max (base 2) and sum.
#pragma unroll
  for (int h = 0; h < GRP; ++h) {
    float *rec = a.partial +
                 ((static_cast<size_t>(b) * a.Hq + g * GRP + h) * a.n_split + s) * (D + 2);
#pragma unroll
    for (int e = 0; e < EPL; ++e) rec[chan<D>(lane, e)] = acc[h][e];
  }
  if (lane < GRP) {
    float *rec = a.partial +
                 ((static_cast<size_t>(b) * a.Hq + g * GRP + lane) * a.n_split + s) * (D + 2);
    rec[D] = m_mine;
    rec[D + 1] = l_mine;
  }
}

// Merge the split partials of one (b, head): one warp per head.
template <int D>
__global__ void __launch_bounds__(128)
decode_combine_kernel(DecodeArgs a) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.x * 4 + warp;
  if (bh >= a.B * a.Hq) return;
  const float *rec = a.partial + static_cast<size_t>(bh) * a.n_split * (D + 2);
  float M = -INFINITY;
  for (int s = lane; s < a.n_split; s += 32) M = fmaxf(M, rec[s * (D + 2) + D]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  float lsum = 0.f;
  for (int s = lane; s < a.n_split; s += 32) {
    const float m = rec[s * (D + 2) + D];
    lsum += rec[s * (D + 2) + D + 1] * exp2f(m - M);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, o);
  constexpr int PER = D / 32;
  float o_acc[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) o_acc[e] = 0.f;
  for (int s = 0; s < a.n_split; ++s) {
    const float w = exp2f(rec[s * (D + 2) + D] - M);
#pragma unroll
    for (int e = 0; e < PER; ++e) o_acc[e] = fmaf(w, rec[s * (D + 2) + lane + 32 * e], o_acc[e]);
  }
  const float inv = 1.f / lsum;
#pragma unroll
  for (int e = 0; e < PER; ++e) {
    const size_t idx = static_cast<size_t>(bh) * D + lane + 32 * e;
    if (a.out_f32)
      reinterpret_cast<float *>(a.out)[idx] = o_acc[e] * inv;
    else
      reinterpret_cast<__nv_bfloat16 *>(a.out)[idx] = __float2bfloat16_rn(o_acc[e] * inv);
  }
  if (lane == 0 && a.lse) a.lse[bh] = (M + log2f(lsum)) * 0.69314718055994531f;
}

template <int D, int GRP>
cudaError_t launch_split(const DecodeArgs &a, cudaStream_t stream) {
  const int smem = DecCfg<D>::BYTES;
  cudaError_t e = cudaFuncSetAttribute(decode_split_kernel<D, GRP>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int n_chunk = (a.Hkv + kDecWarps - 1) / kDecWarps;
  decode_split_kernel<D, GRP><<<dim3(a.n_split, n_chunk, a.B), kDecThreads, smem, stream>>>(a);
  return cudaGetLastError();
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
  const int nbh = a.B * a.Hq;
  decode_combine_kernel<D><<<(nbh + 3) / 4, 128, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace

void decode_plan(int B, int Hkv, int L, int *n_split, int *chunk) {
  // Two CTAs per SM (each holds a 3-stage ring of about 100 KB) over the 148
  // SMs of a B200; chunks are whole stages (8 or 16 tokens).  The split count
  // is non-decreasing in L, so workspace sized for the largest L of a
  // generation loop covers every step.
  const int units = B * ((Hkv + kDecWarps - 1) / kDecWarps);
  int ns = (kCtasPerSm * 148 + units - 1) / units;
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

}  // namespace jl
