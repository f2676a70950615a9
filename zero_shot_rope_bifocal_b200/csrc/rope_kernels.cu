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

// FP16 MMA operand; returns false if a value left the FP16 range.
__device__ __forceinline__ bool store_f16(__half *dst, int i, int half, const Rot2 &v) {
  const __half2 lo = __floats2half2_rn(v.r0, v.r1);
  const __half2 hi = __floats2half2_rn(v.s0, v.s1);
  *reinterpret_cast<__half2 *>(dst + i) = lo;
  *reinterpret_cast<__half2 *>(dst + i + half) = hi;
  return !(__hisinf(__low2half(lo)) | __hisinf(__high2half(lo)) | __hisinf(__low2half(hi)) |
           __hisinf(__high2half(hi)));
}

__global__ void __launch_bounds__(kRopeThreads)
rope_kv_kernel(PrefillArgs a) {
  extern __shared__ float2 cs_smem[];  // [2][kPosPerCta][D/2] (cos, sin), then 2 x [D/2] freq
  const int half = a.D / 2;
  const int b = blockIdx.y;
  const int p_begin = blockIdx.x * kPosPerCta;
  const int npos = min(kPosPerCta, a.L - p_begin);
  const bool two = a.G > 1;
  float2 *cs_true = cs_smem;
  float2 *cs_remote = cs_smem + kPosPerCta * half;

  double *freq = reinterpret_cast<double *>(cs_smem + 2 * kPosPerCta * half);
  double *freq_remote = freq + half;  // theta'_t (interpolation) or theta_t
  const double theta = static_cast<double>(a.theta);
  for (int i = threadIdx.x; i < half; i += blockDim.x) {
    const double f = rope_freq(i, a.D, theta);
    freq[i] = f;
    freq_remote[i] =
        a.interp ? f * interp_factor(f, a.L, a.w_pretrained, a.ramp_alpha, a.ramp_beta) : f;
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < npos * half * (two ? 2 : 1); idx += blockDim.x) {
    const int var = idx / (npos * half);
    const int rem = idx - var * npos * half;
    const int t = rem / half, i = rem - t * half;
    const int pos = p_begin + t;
    const long long ppos = (var == 0 || a.interp) ? pos : remap(pos, a.G);
    float c, s;
    rope_cos_sin(ppos, var == 0 ? freq[i] : freq_remote[i], c, s);
    (var == 0 ? cs_true : cs_remote)[t * half + i] = make_float2(c, s);
  }
  __syncthreads();

  bool in_range = true;
  const int quarter = a.D / 4;  // pairs of channel pairs per head row
  // keys (+ optional true-position cache) and values
  for (int idx = threadIdx.x; idx < npos * a.Hkv * quarter; idx += blockDim.x) {
    const int t = idx / (a.Hkv * quarter);
    const int rem = idx - t * a.Hkv * quarter;
    const int g = rem / quarter;
    const int i = (rem - g * quarter) * 2;
    const int pos = p_begin + t;
    const size_t srow = ((static_cast<size_t>(b) * a.L + pos) * a.Hkv + g) * a.D;
    const __nv_bfloat16 *src = a.k + srow;
    const size_t drow = ((static_cast<size_t>(b) * a.Hkv + g) * a.L + pos) * a.D;
    const Rot2 kt = rotate2(src, i, half, cs_true[t * half + i], cs_true[t * half + i + 1]);
    in_range &= store_f16(a.k_true + drow, i, half, kt);
    if (two)
      in_range &= store_f16(a.k_remote + drow, i, half,
                            rotate2(src, i, half, cs_remote[t * half + i],
                                    cs_remote[t * half + i + 1]));
    if (a.k_cache_out)
      store_bf16(a.k_cache_out + ((static_cast<size_t>(b) * a.k_cache_capacity + pos) * a.Hkv + g) * a.D,
                 i, half, kt);
    // values: the identity rotation, i.e. a BF16 -> FP16 copy into head-major order
    in_range &= store_f16(a.v_op + drow, i, half,
                          rotate2(a.v + srow, i, half, make_float2(1.f, 0.f), make_float2(1.f, 0.f)));
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
cache_kv_kernel(PrefillArgs a) {
  extern __shared__ float2 cs_smem[];  // [kPosPerCta][D/2] (cos, sin), then [D/2] freq
  const int half = a.D / 2;
  const int b = blockIdx.y;
  const int j_begin = blockIdx.x * kPosPerCta;
  const int npos = min(kPosPerCta, a.L - j_begin);
  const bool two = a.G > 1;
  double *freq = reinterpret_cast<double *>(cs_smem + kPosPerCta * half);
  const double theta = static_cast<double>(a.theta);
  for (int i = threadIdx.x; i < half; i += blockDim.x) {
    const double f = rope_freq(i, a.D, theta);
    // the correction's angle per unit of Delta: theta_i, or theta'_i - theta_i
    freq[i] = a.interp ? f * (interp_factor(f, a.L, a.w_pretrained, a.ramp_alpha, a.ramp_beta) - 1.0)
                       : f;
  }
  __syncthreads();
  if (two) {
    for (int idx = threadIdx.x; idx < npos * half; idx += blockDim.x) {
      const int t = idx / half, i = idx - t * half;
      const int j = j_begin + t;
      const long long delta = a.interp ? j : static_cast<long long>(remap(j, a.G)) - j;
      float c, s;
      rope_cos_sin(delta, freq[i], c, s);
      cs_smem[t * half + i] = make_float2(c, s);
    }
  }
  __syncthreads();
  bool in_range = true;
  const int quarter = a.D / 4;
  const float2 one = make_float2(1.f, 0.f);
  for (int idx = threadIdx.x; idx < npos * a.Hkv * quarter; idx += blockDim.x) {
    const int t = idx / (a.Hkv * quarter);
    const int rem = idx - t * a.Hkv * quarter;
    const int g = rem / quarter;
    const int i = (rem - g * quarter) * 2;
    const int j = j_begin + t;
    const size_t srow = ((static_cast<size_t>(b) * a.cache_cap + j) * a.Hkv + g) * a.D;
    const size_t drow = ((static_cast<size_t>(b) * a.Hkv + g) * a.L + j) * a.D;
    const __nv_bfloat16 *kc = a.k_cache_in + srow;
    in_range &= store_f16(a.k_true + drow, i, half, rotate2(kc, i, half, one, one));
    if (two)
      in_range &= store_f16(a.k_remote + drow, i, half,
                            rotate2(kc, i, half, cs_smem[t * half + i], cs_smem[t * half + i + 1]));
    in_range &= store_f16(a.v_op + drow, i, half, rotate2(a.v_cache_in + srow, i, half, one, one));
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

cudaError_t launch_rope_kv(const PrefillArgs &a, cudaStream_t stream) {
  const dim3 grid((a.L + kPosPerCta - 1) / kPosPerCta, a.B);
  const size_t smem = 2 * kPosPerCta * (a.D / 2) * sizeof(float2) + 2 * (a.D / 2) * sizeof(double);
  rope_kv_kernel<<<grid, kRopeThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_chunk_operands(const PrefillArgs &a, cudaStream_t stream) {
  const size_t smem_k = kPosPerCta * (a.D / 2) * sizeof(float2) + (a.D / 2) * sizeof(double);
  cache_kv_kernel<<<dim3((a.L + kPosPerCta - 1) / kPosPerCta, a.B), kRopeThreads, smem_k, stream>>>(a);
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
