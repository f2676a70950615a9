// jl_common.cuh -- definitions shared by the library's translation units:
// the schedule of §3.1, RoPE angle evaluation, bf16 helpers, and the
// launcher interfaces between the C-ABI layer and the kernels.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <climits>
#include <cstdint>

namespace jl {

// Incremented by jetlong_shutdown: host-side caches made before it are stale.
extern std::atomic<unsigned> g_state_epoch;

// Sets a kernel's dynamic shared-memory limit once per device (bit `dev` of a
// per-kernel mask), so later launches make no other CUDA call and can be
// captured into a CUDA graph.  The mask is cleared when jetlong_shutdown has
// run since it was filled (a device reset drops the attribute).
template <auto Kernel>
cudaError_t ensure_smem_limit(int bytes) {
  static std::atomic<unsigned long long> done{0};
  static std::atomic<unsigned> seen_epoch{0};
  const unsigned epoch = g_state_epoch.load(std::memory_order_acquire);
  if (seen_epoch.load(std::memory_order_acquire) != epoch) {
    done.store(0, std::memory_order_release);
    seen_epoch.store(epoch, std::memory_order_release);
  }
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaGetLastError();
  const unsigned long long bit = 1ull << (dev & 63);
  if (done.load(std::memory_order_acquire) & bit) return cudaSuccess;
  const cudaError_t e =
      cudaFuncSetAttribute(Kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) done.fetch_or(bit, std::memory_order_acq_rel);
  return e;
}


// Kernel-side error bits written to the device error word.
enum : unsigned int {
  kDevOk = 0u,
  kDevTimeout = 1u,   // a bounded wait expired
  kDevRange = 2u,     // an operand left the FP16 range of the MMA operands
};

// Time limit for any single in-kernel wait.  Every legitimate wait in these
// kernels (a TMA tile landing, an MMA group finishing) lasts microseconds;
// a quarter of a second means a lost arrival.
constexpr uint64_t kWaitLimitNs = 250000000ull;

// §3.1, Eq. (2): G = max(1, ceil(L / w_pretrained)), integer arithmetic.
__host__ __device__ __forceinline__ int group_size(int L, int w_pretrained) {
  const long long g = (static_cast<long long>(L) + w_pretrained - 1) / w_pretrained;
  return g < 1 ? 1 : static_cast<int>(g);
}

// §3.1: remote position f(x) = floor(x / G) for x >= 0.
__host__ __device__ __forceinline__ int remap(int x, int G) { return x / G; }

// floor(x / G) for 0 <= x < 2^32 by one multiply-high, shift and add
// (Granlund and Montgomery, "Division by invariant integers using
// multiplication", 1994, unsigned case): with l = ceil(log2 G),
// m = floor(2^32 (2^l - G) / G) + 1, t = mulhi(m, x), the quotient is
// (t + ((x - t) >> min(l, 1))) >> max(l - 1, 0).  The kernels use it where
// a division by the run-time G would sit in a per-token loop.
struct GroupDivider {
  uint32_t m;
  int sh1, sh2;
};
inline GroupDivider make_group_divider(int G) {
  int l = 0;
  while ((1ull << l) < static_cast<unsigned long long>(G)) ++l;
  const unsigned long long m =
      ((1ull << 32) * ((1ull << l) - static_cast<unsigned long long>(G))) / static_cast<unsigned long long>(G) + 1ull;
  return GroupDivider{static_cast<uint32_t>(m), l < 1 ? l : 1, l > 1 ? l - 1 : 0};
}
__device__ __forceinline__ int remap_fast(int x, const GroupDivider &dv) {
  const uint32_t u = static_cast<uint32_t>(x);
  const uint32_t t = __umulhi(dv.m, u);
  return static_cast<int>((t + ((u - t) >> dv.sh1)) >> dv.sh2);
}

// RoPE frequency theta^(-2i/D) in double precision.
__device__ __forceinline__ double rope_freq(int i, int D, double theta) {
  return exp(-2.0 * static_cast<double>(i) / static_cast<double>(D) * log(theta));
}

// cos / sin of the RoPE angle pos * freq.  The product is formed in double,
// reduced by the nearest multiple of 2*pi (split into a double head and tail
// so the reduction stays exact to ~1e-16 relative for |angle| < 2^40), and the
// reduced angle in [-pi, pi] goes to the single-precision sine/cosine.
__device__ __forceinline__ void rope_cos_sin(long long pos, double freq, float &c, float &s) {
  const double two_pi_hi = 6.283185307179586232;   // nearest double to 2*pi
  const double two_pi_lo = 2.4492935982947064e-16; // 2*pi - two_pi_hi
  const double a = static_cast<double>(pos) * freq;
  const double n = rint(a * 0.15915494309189533577);  // a / (2*pi), rounded
  double r = fma(-n, two_pi_hi, a);
  r = fma(-n, two_pi_lo, r);
  sincosf(static_cast<float>(r), &s, &c);
}

// Frequency-interpolation remote map (the §4.7 / Table 6 ablation): the
// remote branch scores pairs at their true positions with frequencies
// theta'_t = theta_t * ((1 - gamma_t) / s + gamma_t), YaRN's per-frequency
// ramp gamma_t = clamp((r_t - alpha) / (beta - alpha), 0, 1) over the turns
// r_t = w_pretrained * theta_t / (2 pi) that frequency t makes within the
// pretrained window, and s = max(1, L / w_pretrained), the continuous dynamic
// factor of §3.1.  Returns theta'_t / theta_t.
__host__ __device__ __forceinline__ double interp_factor(double freq, int L, int w_pretrained,
                                                double alpha, double beta) {
  const double s = fmax(1.0, static_cast<double>(L) / static_cast<double>(w_pretrained));
  const double turns = static_cast<double>(w_pretrained) * freq * 0.15915494309189533577;
  const double gam = fmin(1.0, fmax(0.0, (turns - alpha) / (beta - alpha)));
  return (1.0 - gam) / s + gam;
}

__device__ __forceinline__ float bf2f(__nv_bfloat16 x) { return __bfloat162float(x); }

// ---------------------------------------------------------------- launchers
// What one prefill attention launch computes: the fused bifocal rule (§3), or
// one pass of the three-pass inclusion-exclusion merge (§3.3).
enum PrefillPass : int {
  kPassFused = 0,
  kPassRemoteCausal = 1,  // A: remote positions, every causal pair
  kPassLocalBand = 2,     // B: true positions, 0 <= i - j <= w0
  kPassRemoteBand = 3,    // C: remote positions, 0 <= i - j <= w0
};

struct PrefillArgs {
  // caller buffers
  const __nv_bfloat16 *q, *k, *v;
  void *out;
  float *lse;
  int out_f32;
  __nv_bfloat16 *k_cache_out;
  int k_cache_capacity;
  // key operands in the workspace, FP16 head-major [B, Hkv, L, D]: keys
  // rotated to true / remote positions, and the values (the queries are
  // rotated by the attention kernel from q)
  __half *k_true, *k_remote, *v_op;
  // sizes and method parameters; L is the number of keys (positions
  // [0, L)), the queries are positions [q_off, q_off + Lq) with
  // q_off + Lq = L (a whole prompt: q_off = 0, Lq = L)
  int B, Hq, Hkv, L, D, w_pretrained, w0, G;
  int q_off, Lq;
  // keys and values from the true-position cache [B, cache_cap, Hkv, D]
  // instead of pre-RoPE k and v (a chunk appended to a cache)
  const __nv_bfloat16 *k_cache_in, *v_cache_in;
  int cache_cap;
  float theta;
  int pass;  // PrefillPass
  // remote map: 0 = positions aliased by f (the method), 1 = frequency
  // interpolation with ramp bounds (ramp_alpha, ramp_beta) (the ablation)
  int interp;
  float ramp_alpha, ramp_beta;
  unsigned int *dev_error;
  // Key split (a chunk with few query tiles): n_split > 1 splits each query
  // tile's key visits into n_split contiguous ranges, one CTA each, which
  // write unnormalised partial records [B, Lq, Hq, n_split, D + 2] (O, the
  // base-2 max, the sum) to `partial`; launch_split_merge then forms out and
  // lse.  n_split = 1: the kernel writes out and lse itself.
  int n_split;
  float *partial;
  // Turns per position as 64-bit binary fractions, formed on the host by the
  // key-pass launchers: theta_i / (2 pi) (omega_true), the remote map's
  // (theta_i, or theta'_i under the interpolation map), and the correction
  // rotation's per unit of Delta (theta_i, or theta'_i - theta_i, negative,
  // in two's complement).
  uint64_t omega_true[64], omega_remote[64], omega_corr[64];
};

// Rotates k into the two key operand arrays, copies v to its operand array
// (and writes the optional cache).
cudaError_t launch_rope_kv(const PrefillArgs &a, cudaStream_t stream);

// The key operands of a chunk appended to a cache: the cached keys and values
// of positions [0, L) as FP16 operands, the keys also in their remote form
// (the correction rotation of §3.2 applied).
cudaError_t launch_chunk_operands(const PrefillArgs &a, cudaStream_t stream);

// The attention kernel proper (tcgen05 / TMEM / TMA).
cudaError_t launch_prefill_attention(const PrefillArgs &a, cudaStream_t stream);

// out = (W_A O_A + W_B O_B - W_C O_C) / (W_A + W_B - W_C), W_X = exp(lse_X),
// over the three passes' fp32 outputs [B, L, Hq, D] and lse [B, Hq, L].
cudaError_t launch_three_pass_merge(const float *o_a, const float *o_b, const float *o_c,
                                    const float *l_a, const float *l_b, const float *l_c,
                                    void *out, float *lse, int out_f32, int B, int Hq, int L,
                                    int D, cudaStream_t stream);

struct DecodeArgs {
  const __nv_bfloat16 *q, *k_cache, *v_cache;
  // Remote form of the key cache, FP16 R(f(j) - j) k_cache[j] for the call's
  // G (same layout as k_cache), or NULL: then remote keys are turned on the fly.
  const __half *k_remote;
  void *out;
  float *lse;
  int out_f32;
  float *partial;  // workspace: [B, Hq, n_split, D + 2]
  int B, Hq, Hkv, L, Lcap, D, w_pretrained, w0, G;
  float theta;
  int n_split, chunk;
  // Queries per batch entry and the position of the first: a decode step has
  // nq = 1 at q_pos0 = L - 1; a prefill chunk has nq = n at q_pos0 = P0, and
  // query i sees keys [0, q_pos0 + i].  q is [B, nq, Hq, D], out likewise,
  // lse [B, Hq, nq]; L is the longest key range, q_pos0 + nq.
  int nq, q_pos0;
  int interp;  // remote map, as in PrefillArgs
  float ramp_alpha, ramp_beta;
  GroupDivider gdiv;  // floor(x / G) by multiplication
  // Turns per position as 64-bit binary fractions (theta_i / (2 pi)), formed
  // on the host: of the true query (omega_qt), of the remote query (at f(p)
  // with theta_i, or at p with theta'_i under the interpolation map), and of
  // the correction rotation per unit of Delta (theta_i, or theta'_i - theta_i,
  // negative, in two's complement).
  uint64_t omega_qt[64], omega_qr[64], omega_corr[64];
  unsigned int *dev_error;
};

// Split-KV plan: number of key chunks and chunk length for a cache of L tokens.
void decode_plan(int B, int Hkv, int L, int *n_split, int *chunk);

// Query heads per KV head (Hq / Hkv) the decode kernel is built for: 1, 2, 4, 8.
bool decode_supports_group(int grp);

cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t stream);

// Log-sum-exp merge of split partial records [B, nq, Hq, n_split, D + 2]
// (unnormalised O, base-2 max, sum) into out [B, nq, Hq, D] and lse
// [B, Hq, nq] (lse may be NULL); n_split <= 296.
cudaError_t launch_split_merge(const float *partial, int n_split, void *out, int out_f32,
                               float *lse, int B, int nq, int Hq, int D, cudaStream_t stream);

// k_remote[b, j] = FP16(R(f(j) - j) k_cache[b, j]) for j in [j0, j1), all KV heads.
cudaError_t launch_remote_cache(const __nv_bfloat16 *k_cache, __half *k_remote, int B, int Lcap,
                                int Hkv, int D, int j0, int j1, int G, float theta,
                                cudaStream_t stream);

cudaError_t launch_rope_cache(const __nv_bfloat16 *k, __nv_bfloat16 *k_cache, int B, int n,
                              int Hkv, int D, int pos0, int Lcap, float theta,
                              cudaStream_t stream);

}  // namespace jl
