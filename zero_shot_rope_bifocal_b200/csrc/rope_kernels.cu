// rope_kernels.cu -- the key side of RoPE for the bifocal attention (the
// queries are rotated in the attention kernel's load path, see
// prefill_sm100.cu).
//
// Prefill key operands (Jet-Long paper, §3 score rule and §3.2): every key
// is rotated to its true position j and to its remote position f(j):
//
//   k_true[b,g,j]  = RoPE(x_k, j)      k_remote[b,g,j] = RoPE(x_k, f(j))
//
// k_true is exactly the true-position KV cache of §3.2, and k_remote equals
// the correction rotation by Delta j = f(j) - j applied to it.  The outputs
// (and a copy of v) are the tensor-core operands: FP16, head-major
// [B, Hkv, L, D], so that the attention kernel's TMA fetches each 128-token
// tile as one contiguous block.  Every key tile is read by every query tile
// of its KV head, so the keys are rotated once here rather than in each
// CTA.  FP16 holds the rotated values with three more mantissa bits than
// BF16; a value beyond the FP16 range (|x| > 65504) is reported through the
// device error word.  The optional cache output keeps the caller's BF16
// format.  When G == 1 (L <= w_pretrained, the native-window case of
// Appendix H) f is the identity and only the true-position arrays are
// written.
//
// With the frequency-interpolation remote map (the §4.7 ablation) the remote
// arrays hold RoPE'(x, j): true position, interpolated frequencies theta'_t.
//
// Chunk operands (a chunk of queries appended to a cache, §3.1, §3.2): the
// keys and values read from the true-position cache; the remote keys are the
// cached ones turned by the correction rotation R(f(j) - j).
//
// Cache writer (§3.2): k_cache[b, pos0 + t] = RoPE(k[b, t], pos0 + t).
//
// Each CTA forms the frequencies once, evaluates cos/sin once per (position,
// frequency) into shared memory and applies it to every head of that
// position; channel pairs are (i, i + D/2), processed two pairs per thread
// with BF16x2 loads and FP16x2 stores.
#include <cmath>

#include "jl_common.cuh"

namespace jl {
namespace {

constexpr int kRopeThreads = 256;
constexpr int kPosPerCta = 8;

// Rotated pairs (a[i], a[i+D/2]) and (a[i+1], a[i+1+D/2]) of one BF16 head row,
// in fp32: returns (r0, r1) for channels i, i+1 and (s0, s1) for i+D/2, i+1+D/2.
struct Rot2 {
  float r0, r1, s0, s1;
};

__device__ __forceinline__ Rot2 rotate2(const __nv_bfloat16 *src, int i, int half, float2 cs0,
                                        float2 cs1) {
  const __nv_bfloat162 lo = *reinterpret_cast<const __nv_bfloat162 *>(src + i);
  const __nv_bfloat162 hi = *reinterpret_cast<const __nv_bfloat162 *>(src + i + half);
  const float a0 = __low2float(lo), a1 = __high2float(lo);
  const float b0 = __low2float(hi), b1 = __high2float(hi);
  // cs = (cos, sin)
  return {a0 * cs0.x - b0 * cs0.y, a1 * cs1.x - b1 * cs1.y, a0 * cs0.y + b0 * cs0.x,
          a1 * cs1.y + b1 * cs1.x};
}

__device__ __forceinline__ void store_bf16(__nv_bfloat16 *dst, int i, int half, const Rot2 &v) {
  *reinterpret_cast<__nv_bfloat162 *>(dst + i) = __floats2bfloat162_rn(v.r0, v.r1);
  *reinterpret_cast<__nv_bfloat162 *>(dst + i + half) = __floats2bfloat162_rn(v.s0, v.s1);
}

// Positions per CTA of the key passes; every position's (cos, sin) is formed
// once and used by every KV head.
constexpr int kKvPos = 16;
constexpr float kTurnToRad = 1.4629180792671596e-09f;  // 2 pi / 2^32

// cos / sin of the angle whose turns are (pos * omega) mod 1, exact in
// 64-bit fixed point: the wrapping product's top 32 bits are the signed
// phase, so the sine/cosine only sees [-pi, pi).
__device__ __forceinline__ float2 turn_cos_sin(uint64_t pos, uint64_t omega) {
  const int32_t ph = static_cast<int32_t>((pos * omega) >> 32);
  float c, s;
  __sincosf(static_cast<float>(ph) * kTurnToRad, &s, &c);
  return make_float2(c, s);
}

// Eight channel pairs (c .. c+7 with partners c+D/2 ..) of a BF16 row,
// loaded as two 16-byte vectors, turned by their (cos, sin) and returned as
// FP32 (lo = channels c.., hi = partners).
struct Rot8 {
  float lo[8], hi[8];
};
__device__ __forceinline__ Rot8 rotate8(uint4 xa, uint4 xb, const float2 *cs) {
  const uint32_t wa[4] = {xa.x, xa.y, xa.z, xa.w}, wb[4] = {xb.x, xb.y, xb.z, xb.w};
  Rot8 r;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const uint32_t ua = wa[e >> 1], ub = wb[e >> 1];
    const float x = __uint_as_float((e & 1) ? (ua & 0xffff0000u) : (ua << 16));
    const float y = __uint_as_float((e & 1) ? (ub & 0xffff0000u) : (ub << 16));
    r.lo[e] = x * cs[e].x - y * cs[e].y;
    r.hi[e] = x * cs[e].y + y * cs[e].x;
  }
  return r;
}

// Stores 8 values as FP16 (16 bytes); returns false if one left the FP16 range.
__device__ __forceinline__ bool store8_f16(__half *dst, const float (&v)[8]) {
  uint32_t w[4];
  bool ok = true;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const __half2 h = __floats2half2_rn(v[2 * e], v[2 * e + 1]);
    ok &= !(__hisinf(__low2half(h)) | __hisinf(__high2half(h)));
    w[e] = *reinterpret_cast<const uint32_t *>(&h);
  }
  *reinterpret_cast<uint4 *>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
  return ok;
}

__device__ __forceinline__ void store8_bf16(__nv_bfloat16 *dst, const float (&v)[8]) {
  uint32_t w[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * e], v[2 * e + 1]);
    w[e] = *reinterpret_cast<const uint32_t *>(&h);
  }
  *reinterpret_cast<uint4 *>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
}

// BF16 -> FP16 copy of 8 values (the values' operand); false if out of range.
__device__ __forceinline__ bool copy8_f16(__half *dst, uint4 x) {
  const uint32_t w[4] = {x.x, x.y, x.z, x.w};
  float v[8];
#pragma unroll
  for (int e = 0; e < 8; ++e)
    v[e] = __uint_as_float((e & 1) ? (w[e >> 1] & 0xffff0000u) : (w[e >> 1] << 16));
  return store8_f16(dst, v);
}

// Prefill key operands: for each position j of [16 blockIdx.x, +16) and KV
// head g, k_true = RoPE(x_k, j), k_remote = RoPE(x_k, f(j)) (RoPE'(x_k, j)
// under the interpolation map), v copied, all FP16 head-major, plus the
// optional BF16 true-position cache.  Work item = (position, head, group of
// 8 channels and their partners): 16-byte loads and stores.
__global__ void __launch_bounds__(kRopeThreads)
rope_kv_kernel(const __grid_constant__ PrefillArgs a) {
  __shared__ float2 cs[2][kKvPos][64];  // (cos, sin): true, remote
  __shared__ uint64_t om[2][64];
  const int half = a.D / 2;
  const int b = blockIdx.y;
  const int p_begin = blockIdx.x * kKvPos;
  const int npos = min(kKvPos, a.L - p_begin);
  const bool two = a.G > 1;
  if (threadIdx.x < half) {
    om[0][threadIdx.x] = a.omega_true[threadIdx.x];
    om[1][threadIdx.x] = a.omega_remote[threadIdx.x];
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < npos * half * (two ? 2 : 1); idx += blockDim.x) {
    const int var = idx / (npos * half);
    const int rem = idx - var * npos * half;
    const int t = rem / half, i = rem - t * half;
    const int pos = p_begin + t;
    const uint64_t pp = (var == 0 || a.interp) ? pos : remap(pos, a.G);
    cs[var][t][i] = turn_cos_sin(pp, om[var][i]);
  }
  __syncthreads();
  bool in_range = true;
  const int c8n = a.D / 16;  // groups of 8 channel pairs per head row
  for (int idx = threadIdx.x; idx < npos * a.Hkv * c8n; idx += blockDim.x) {
    const int t = idx / (a.Hkv * c8n);
    const int rem = idx - t * a.Hkv * c8n;
    const int g = rem / c8n;
    const int c = (rem - g * c8n) * 8;
    const int pos = p_begin + t;
    const size_t srow = ((static_cast<size_t>(b) * a.L + pos) * a.Hkv + g) * a.D;
    const size_t drow = ((static_cast<size_t>(b) * a.Hkv + g) * a.L + pos) * a.D;
    const uint4 ka = __ldg(reinterpret_cast<const uint4 *>(a.k + srow + c));
    const uint4 kb = __ldg(reinterpret_cast<const uint4 *>(a.k + srow + c + half));
    const Rot8 kt = rotate8(ka, kb, &cs[0][t][c]);
    in_range &= store8_f16(a.k_true + drow + c, kt.lo);
    in_range &= store8_f16(a.k_true + drow + c + half, kt.hi);
    if (two) {
      const Rot8 kr = rotate8(ka, kb, &cs[1][t][c]);
      in_range &= store8_f16(a.k_remote + drow + c, kr.lo);
      in_range &= store8_f16(a.k_remote + drow + c + half, kr.hi);
    }
    if (a.k_cache_out) {
      __nv_bfloat16 *crow =
          a.k_cache_out + ((static_cast<size_t>(b) * a.k_cache_capacity + pos) * a.Hkv + g) * a.D;
      store8_bf16(crow + c, kt.lo);
      store8_bf16(crow + c + half, kt.hi);
    }
    in_range &= copy8_f16(a.v_op + drow + c, __ldg(reinterpret_cast<const uint4 *>(a.v + srow + c)));
    in_range &= copy8_f16(a.v_op + drow + c + half,
                          __ldg(reinterpret_cast<const uint4 *>(a.v + srow + c + half)));
  }
  if (!in_range) atomicOr(a.dev_error, kDevRange);
}

// Chunk operands, keys and values from the true-position cache (§3.2): for
// j < L,
//   k_true[b,g,j] = k_cache[b,j,g],  k_remote[b,g,j] = R(f(j) - j) k_cache[b,j,g],
//   v_op[b,g,j] = v_cache[b,j,g],
// FP16 head-major [B, Hkv, L, D].  R(Delta) turns channel pair (i, i + D/2) by
// Delta * theta_i; under the frequency-interpolation map the remote form is
// RoPE'(x_k, j), i.e. the cached key turned by j * (theta'_i - theta_i).
__global__ void __launch_bounds__(kRopeThreads)
cache_kv_kernel(const __grid_constant__ PrefillArgs a) {
  __shared__ float2 cs[kKvPos][64];  // (cos, sin) of the correction
  __shared__ uint64_t om[64];
  const int half = a.D / 2;
  const int b = blockIdx.y;
  const int j_begin = blockIdx.x * kKvPos;
  const int npos = min(kKvPos, a.L - j_begin);
  const bool two = a.G > 1;
  if (threadIdx.x < half) om[threadIdx.x] = a.omega_corr[threadIdx.x];
  __syncthreads();
  if (two) {
    for (int idx = threadIdx.x; idx < npos * half; idx += blockDim.x) {
      const int t = idx / half, i = idx - t * half;
      const int j = j_begin + t;
      const long long delta = a.interp ? j : static_cast<long long>(remap(j, a.G)) - j;
      cs[t][i] = turn_cos_sin(static_cast<uint64_t>(delta), om[i]);
    }
  }
  __syncthreads();
  bool in_range = true;
  const int c8n = a.D / 16;
  const float2 one[8] = {make_float2(1.f, 0.f), make_float2(1.f, 0.f), make_float2(1.f, 0.f),
                         make_float2(1.f, 0.f), make_float2(1.f, 0.f), make_float2(1.f, 0.f),
                         make_float2(1.f, 0.f), make_float2(1.f, 0.f)};
  for (int idx = threadIdx.x; idx < npos * a.Hkv * c8n; idx += blockDim.x) {
    const int t = idx / (a.Hkv * c8n);
    const int rem = idx - t * a.Hkv * c8n;
    const int g = rem / c8n;
    const int c = (rem - g * c8n) * 8;
    const int j = j_begin + t;
    const size_t srow = ((static_cast<size_t>(b) * a.cache_cap + j) * a.Hkv + g) * a.D;
    const size_t drow = ((static_cast<size_t>(b) * a.Hkv + g) * a.L + j) * a.D;
    const uint4 ka = __ldg(reinterpret_cast<const uint4 *>(a.k_cache_in + srow + c));
    const uint4 kb = __ldg(reinterpret_cast<const uint4 *>(a.k_cache_in + srow + c + half));
    const Rot8 kt = rotate8(ka, kb, one);
    in_range &= store8_f16(a.k_true + drow + c, kt.lo);
    in_range &= store8_f16(a.k_true + drow + c + half, kt.hi);
    if (two) {
      const Rot8 kr = rotate8(ka, kb, &cs[t][c]);
      in_range &= store8_f16(a.k_remote + drow + c, kr.lo);
      in_range &= store8_f16(a.k_remote + drow + c + half, kr.hi);
    }
    in_range &= copy8_f16(a.v_op + drow + c,
                          __ldg(reinterpret_cast<const uint4 *>(a.v_cache_in + srow + c)));
    in_range &= copy8_f16(a.v_op + drow + c + half,
                          __ldg(reinterpret_cast<const uint4 *>(a.v_cache_in + srow + c + half)));
  }
  if (!in_range) atomicOr(a.dev_error, kDevRange);
}

__global__ void __launch_bounds__(kRopeThreads)
rope_cache_kernel(const __nv_bfloat16 *__restrict__ k, __nv_bfloat16 *__restrict__ k_cache, int n,
                  int Hkv, int D, int pos0, int Lcap, float theta_f) {
  extern __shared__ float2 cs_smem[];  // [kPosPerCta][D/2], then [D/2] freq
  const int half = D / 2;
  const int b = blockIdx.y;
  const int t_begin = blockIdx.x * kPosPerCta;
  const int npos = min(kPosPerCta, n - t_begin);
  double *freq = reinterpret_cast<double *>(cs_smem + kPosPerCta * half);
  const double theta = static_cast<double>(theta_f);
  for (int i = threadIdx.x; i < half; i += blockDim.x) freq[i] = rope_freq(i, D, theta);
  __syncthreads();
  for (int idx = threadIdx.x; idx < npos * half; idx += blockDim.x) {
    const int t = idx / half, i = idx - t * half;
    float c, s;
    rope_cos_sin(static_cast<long long>(pos0) + t_begin + t, freq[i], c, s);
    cs_smem[t * half + i] = make_float2(c, s);
  }
  __syncthreads();
  const int quarter = D / 4;
  for (int idx = threadIdx.x; idx < npos * Hkv * quarter; idx += blockDim.x) {
    const int t = idx / (Hkv * quarter);
    const int rem = idx - t * Hkv * quarter;
    const int g = rem / quarter;
    const int i = (rem - g * quarter) * 2;
    const __nv_bfloat16 *src = k + ((static_cast<size_t>(b) * n + t_begin + t) * Hkv + g) * D;
    __nv_bfloat16 *dst =
        k_cache + ((static_cast<size_t>(b) * Lcap + pos0 + t_begin + t) * Hkv + g) * D;
    store_bf16(dst, i, half, rotate2(src, i, half, cs_smem[t * half + i], cs_smem[t * half + i + 1]));
  }
}

}  // namespace

// The key passes' turn fractions for the call's theta, map and length.
static PrefillArgs with_turns(const PrefillArgs &a) {
  PrefillArgs t = a;
  const double turns_q64 = 0.15915494309189533577 * 18446744073709551616.0;  // 2^64 / (2 pi)
  const double log_theta = std::log(static_cast<double>(a.theta));
  for (int i = 0; i < a.D / 2; ++i) {
    const double f = std::exp(-2.0 * static_cast<double>(i) / static_cast<double>(a.D) * log_theta);
    const double factor =
        a.interp ? interp_factor(f, a.L, a.w_pretrained, a.ramp_alpha, a.ramp_beta) : 1.0;
    t.omega_true[i] = static_cast<uint64_t>(std::llround(f * turns_q64));  // < 2^62
    t.omega_remote[i] = static_cast<uint64_t>(std::llround(f * factor * turns_q64));
    // (theta' - theta) / (2 pi) lies in (-1/(2 pi), 0]: inside int64 once scaled
    t.omega_corr[i] = a.interp ? static_cast<uint64_t>(std::llround(f * (factor - 1.0) * turns_q64))
                               : t.omega_true[i];
  }
  return t;
}

cudaError_t launch_rope_kv(const PrefillArgs &a, cudaStream_t stream) {
  const dim3 grid((a.L + kKvPos - 1) / kKvPos, a.B);
  rope_kv_kernel<<<grid, kRopeThreads, 0, stream>>>(with_turns(a));
  return cudaGetLastError();
}

cudaError_t launch_chunk_operands(const PrefillArgs &a, cudaStream_t stream) {
  const dim3 grid((a.L + kKvPos - 1) / kKvPos, a.B);
  cache_kv_kernel<<<grid, kRopeThreads, 0, stream>>>(with_turns(a));
  return cudaGetLastError();
}

cudaError_t launch_rope_cache(const __nv_bfloat16 *k, __nv_bfloat16 *k_cache, int B, int n,
                              int Hkv, int D, int pos0, int Lcap, float theta,
                              cudaStream_t stream) {
  const dim3 grid((n + kPosPerCta - 1) / kPosPerCta, B);
  const size_t smem = kPosPerCta * (D / 2) * sizeof(float2) + (D / 2) * sizeof(double);
  rope_cache_kernel<<<grid, kRopeThreads, smem, stream>>>(k, k_cache, n, Hkv, D, pos0, Lcap, theta);
  return cudaGetLastError();
}

}  // namespace jl
