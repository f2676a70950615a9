// decode_kernels.cu -- one generation step of bifocal attention on the
// true-position KV cache (Jet-Long paper, §3.2 "Key-value cache management and
// correction rotation"; score rule of §3; schedule of §3.1 with L = tokens in
// the cache including the new one, query at p = L - 1).
//
// Split-KV: the key range [0, L) is cut into n_split chunks; CTA (s, g, b)
// streams chunk s of KV head g for every query head of that group and keeps
// an online softmax per head.  Keys with p - j <= w0 are scored as cached
// against RoPE(x_q, p); older keys are rotated in shared memory by
// Delta j = f(j) - j (the correction rotation, so the cache is never
// rewritten) and scored against RoPE(x_q, f(p)).  Each CTA writes its
// unnormalised partial output with its running max and sum to the workspace;
// a second kernel merges the partials by log-sum-exp, one warp per head.
//
// Traffic: the kernel reads K and V once (2 * L * Hkv * D * 2 bytes per
// token); everything else is O(Hq * D * n_split).
#include <cmath>

#include "jl_common.cuh"

namespace jl {
namespace {

constexpr int kDecThreads = 128;
constexpr int kKeyBlock = 64;
constexpr int kMaxGrp = 16;
constexpr float kLog2e = 1.4426950408889634f;

template <int D>
struct DecodeSmem {
  static constexpr int KS = D + 4;  // padded fp32 row of K (bank-conflict free float4 reads)
  static size_t bytes(int grp) {
    return sizeof(float) * (2 * grp * D + kKeyBlock * KS + kKeyBlock * D + grp * kKeyBlock +
                            3 * grp) +
           sizeof(double) * (D / 2) + 16;
  }
};

template <int D>
__global__ void __launch_bounds__(kDecThreads)
decode_split_kernel(DecodeArgs a) {
  constexpr int KS = DecodeSmem<D>::KS;
  constexpr int HALF = D / 2;
  const int s = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int grp = a.Hq / a.Hkv;
  const int p = a.L - 1;
  const int G = a.G;
  const int fp = remap(p, G);
  const int w0eff = (G == 1) ? INT_MAX : a.w0;
  const int j_begin = s * a.chunk;
  const int j_end = min(a.L, j_begin + a.chunk);

  extern __shared__ __align__(16) unsigned char dsm[];
  double *freq = reinterpret_cast<double *>(dsm);
  float *q_true = reinterpret_cast<float *>(dsm + sizeof(double) * HALF);  // [grp][D]
  float *q_rem = q_true + grp * D;                                         // [grp][D]
  float *Ks = q_rem + grp * D;                                             // [kKeyBlock][KS]
  float *Vs = Ks + kKeyBlock * KS;                                         // [kKeyBlock][D]
  float *sc = Vs + kKeyBlock * D;                                          // [grp][kKeyBlock]
  float *m_run = sc + grp * kKeyBlock;                                     // [grp]
  float *l_run = m_run + grp;
  float *alpha = l_run + grp;

  const double theta = static_cast<double>(a.theta);
  for (int i = tid; i < HALF; i += kDecThreads) freq[i] = rope_freq(i, D, theta);
  for (int h = tid; h < grp; h += kDecThreads) {
    m_run[h] = -INFINITY;
    l_run[h] = 0.f;
  }
  __syncthreads();

  // Queries at the true position p and the remote position f(p), pre-scaled by
  // log2(e)/sqrt(D) so the softmax runs in base 2.
  const float qscale = kLog2e / sqrtf(static_cast<float>(D));
  for (int idx = tid; idx < grp * HALF; idx += kDecThreads) {
    const int h = idx / HALF, i = idx - h * HALF;
    const __nv_bfloat16 *qrow = a.q + (static_cast<size_t>(b) * a.Hq + g * grp + h) * D;
    const float x = bf2f(qrow[i]), y = bf2f(qrow[i + HALF]);
    float c, sn;
    rope_cos_sin(p, freq[i], c, sn);
    q_true[h * D + i] = (x * c - y * sn) * qscale;
    q_true[h * D + i + HALF] = (x * sn + y * c) * qscale;
    rope_cos_sin(fp, freq[i], c, sn);
    q_rem[h * D + i] = (x * c - y * sn) * qscale;
    q_rem[h * D + i + HALF] = (x * sn + y * c) * qscale;
  }

  constexpr int kMaxOut = kMaxGrp * D / kDecThreads;
  float acc[kMaxOut];
#pragma unroll
  for (int r = 0; r < kMaxOut; ++r) acc[r] = 0.f;
  const int n_out = grp * D;

  const size_t row_stride = static_cast<size_t>(a.Hkv) * D;
  const __nv_bfloat16 *kbase = a.k_cache + (static_cast<size_t>(b) * a.Lcap * a.Hkv + g) * D;
  const __nv_bfloat16 *vbase = a.v_cache + (static_cast<size_t>(b) * a.Lcap * a.Hkv + g) * D;

  for (int jb = j_begin; jb < j_end; jb += kKeyBlock) {
    const int nk = min(kKeyBlock, j_end - jb);
    __syncthreads();  // previous block fully consumed
    // Stage K and V rows (8 BF16 per 16-byte load) as fp32.
    for (int idx = tid; idx < kKeyBlock * (D / 8); idx += kDecThreads) {
      const int t = idx / (D / 8), c8 = (idx - t * (D / 8)) * 8;
      float kv[8], vv[8];
      if (t < nk) {
        const uint4 kr = *reinterpret_cast<const uint4 *>(kbase + (jb + t) * row_stride + c8);
        const uint4 vr = *reinterpret_cast<const uint4 *>(vbase + (jb + t) * row_stride + c8);
        const __nv_bfloat162 *k2 = reinterpret_cast<const __nv_bfloat162 *>(&kr);
        const __nv_bfloat162 *v2 = reinterpret_cast<const __nv_bfloat162 *>(&vr);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          kv[2 * e] = __low2float(k2[e]);
          kv[2 * e + 1] = __high2float(k2[e]);
          vv[2 * e] = __low2float(v2[e]);
          vv[2 * e + 1] = __high2float(v2[e]);
        }
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) kv[e] = vv[e] = 0.f;
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        Ks[t * KS + c8 + e] = kv[e];
        Vs[t * D + c8 + e] = vv[e];
      }
    }
    __syncthreads();
    // Correction rotation of the remote keys (p - j > w0): R(Delta j), Delta j = f(j) - j.
    if (p - jb > w0eff) {
      for (int idx = tid; idx < nk * HALF; idx += kDecThreads) {
        const int t = idx / HALF, i = idx - t * HALF;
        const int j = jb + t;
        if (p - j > w0eff) {
          float c, sn;
          rope_cos_sin(static_cast<long long>(remap(j, G)) - j, freq[i], c, sn);
          const float x = Ks[t * KS + i], y = Ks[t * KS + i + HALF];
          Ks[t * KS + i] = x * c - y * sn;
          Ks[t * KS + i + HALF] = x * sn + y * c;
        }
      }
      __syncthreads();
    }
    // Scores for (key t, head h).
    for (int idx = tid; idx < kKeyBlock * grp; idx += kDecThreads) {
      const int t = idx % kKeyBlock, h = idx / kKeyBlock;
      const int j = jb + t;
      float sres = -INFINITY;
      if (t < nk) {
        const float *qv = (p - j > w0eff) ? q_rem + h * D : q_true + h * D;
        const float *kv = Ks + t * KS;
        float acc0 = 0.f, acc1 = 0.f, acc2 = 0.f, acc3 = 0.f;
#pragma unroll 8
        for (int d = 0; d < D; d += 4) {
          const float4 k4 = *reinterpret_cast<const float4 *>(kv + d);
          const float4 q4 = *reinterpret_cast<const float4 *>(qv + d);
          acc0 = fmaf(k4.x, q4.x, acc0);
          acc1 = fmaf(k4.y, q4.y, acc1);
          acc2 = fmaf(k4.z, q4.z, acc2);
          acc3 = fmaf(k4.w, q4.w, acc3);
        }
        sres = (acc0 + acc1) + (acc2 + acc3);
      }
      sc[h * kKeyBlock + t] = sres;
    }
    __syncthreads();
    // Online softmax per head (one warp per head).
    for (int h = warp; h < grp; h += kDecThreads / 32) {
      float v0 = sc[h * kKeyBlock + lane], v1 = sc[h * kKeyBlock + lane + 32];
      float mx = fmaxf(v0, v1);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      const float m_old = m_run[h];
      const float m_new = fmaxf(m_old, mx);  // finite: every block holds a valid key
      const float e0 = exp2f(v0 - m_new), e1 = exp2f(v1 - m_new);
      sc[h * kKeyBlock + lane] = e0;
      sc[h * kKeyBlock + lane + 32] = e1;
      float sum = e0 + e1;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      __syncwarp();
      if (lane == 0) {
        const float al = exp2f(m_old - m_new);  // 0 when m_old = -inf
        alpha[h] = al;
        l_run[h] = l_run[h] * al + sum;
        m_run[h] = m_new;
      }
    }
    __syncthreads();
    // O[h, d] = alpha[h] * O[h, d] + sum_t p[h, t] V[t, d]
#pragma unroll
    for (int r = 0; r < kMaxOut; ++r) {
      const int o = tid + r * kDecThreads;
      if (o < n_out) {
        const int h = o / D, d = o - h * D;
        const float *ph = sc + h * kKeyBlock;
        float x = acc[r] * alpha[h];
#pragma unroll 8
        for (int t = 0; t < kKeyBlock; ++t) x = fmaf(ph[t], Vs[t * D + d], x);
        acc[r] = x;
      }
    }
  }
  __syncthreads();
  // Partial record: [D] unnormalised output, then the running max (base 2) and sum.
#pragma unroll
  for (int r = 0; r < kMaxOut; ++r) {
    const int o = tid + r * kDecThreads;
    if (o < n_out) {
      const int h = o / D, d = o - h * D;
      float *rec = a.partial + ((static_cast<size_t>(b) * a.Hq + g * grp + h) * a.n_split + s) * (D + 2);
      rec[d] = acc[r];
      if (d == 0) {
        rec[D] = m_run[h];
        rec[D + 1] = l_run[h];
      }
    }
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

template <int D>
cudaError_t launch_decode_d(const DecodeArgs &a, cudaStream_t stream) {
  const int grp = a.Hq / a.Hkv;
  const size_t smem = DecodeSmem<D>::bytes(grp);
  cudaError_t e = cudaFuncSetAttribute(decode_split_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  decode_split_kernel<D><<<dim3(a.n_split, a.Hkv, a.B), kDecThreads, smem, stream>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int nbh = a.B * a.Hq;
  decode_combine_kernel<D><<<(nbh + 3) / 4, 128, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace

void decode_plan(int B, int Hkv, int L, int *n_split, int *chunk) {
  // Aim for about four resident CTAs per SM over the 148 SMs of a B200; the
  // split count is non-decreasing in L, so workspace sized for the largest L
  // of a generation loop covers every step.
  const int target = 4 * 148;
  const int units = B * Hkv;
  int ns = (target + units - 1) / units;
  const int max_ns = (L + kKeyBlock - 1) / kKeyBlock;
  if (ns > max_ns) ns = max_ns;
  if (ns < 1) ns = 1;
  int ch = (L + ns - 1) / ns;
  ch = (ch + kKeyBlock - 1) / kKeyBlock * kKeyBlock;
  *chunk = ch;
  *n_split = (L + ch - 1) / ch;
}

int decode_max_group() { return kMaxGrp; }

cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t stream) {
  if (a.D == 128) return launch_decode_d<128>(a, stream);
  return launch_decode_d<64>(a, stream);
}

}  // namespace jl
