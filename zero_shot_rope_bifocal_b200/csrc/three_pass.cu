// three_pass.cu -- the merge step of the unfused three-pass form of bifocal
// attention (Jet-Long paper, §3.3 "Inclusion-exclusion merge").
//
// The three passes are ordinary FlashAttention-style launches of the prefill
// kernel (see PrefillPass): A = attention at remote positions over every
// causal pair, B = attention at true positions over the band 0 <= i - j <= w0,
// C = attention at remote positions over the same band.  Their softmax
// denominators are W_X = exp(lse_X), so the bifocal row is
//   out = (W_A O_A + W_B O_B - W_C O_C) / (W_A + W_B - W_C),
//   lse = log(W_A + W_B - W_C),
// which this kernel forms with the weights taken relative to the largest lse.
// The subtraction is where the unfused form loses precision: its error grows
// with (W_A + W_C) / (W_A + W_B - W_C).  The fused kernel has no subtraction.
//
// Traffic: three fp32 rows in, one row out per (b, i, h); HBM-bound.
#include "jl_common.cuh"

namespace jl {
namespace {

constexpr int kMergeWarps = 8;

// One warp per (b, i, h) row (rows ordered [b][i][h] like the outputs); lanes
// cover the D channels four at a time.
__global__ void __launch_bounds__(kMergeWarps * 32)
three_pass_merge_kernel(const float *__restrict__ o_a, const float *__restrict__ o_b,
                        const float *__restrict__ o_c, const float *__restrict__ l_a,
                        const float *__restrict__ l_b, const float *__restrict__ l_c, void *out,
                        float *lse, int out_f32, int B, int Hq, int L, int D) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long row = static_cast<long long>(blockIdx.x) * kMergeWarps + warp;
  if (row >= static_cast<long long>(B) * L * Hq) return;
  const int h = static_cast<int>(row % Hq);
  const long long bi = row / Hq;
  const int i = static_cast<int>(bi % L);
  const int b = static_cast<int>(bi / L);
  const size_t li = (static_cast<size_t>(b) * Hq + h) * L + i;
  const float la = l_a[li], lb = l_b[li], lc = l_c[li];
  const float M = fmaxf(la, fmaxf(lb, lc));
  const float wa = expf(la - M), wb = expf(lb - M), wc = expf(lc - M);
  const float den = wa + wb - wc;
  const float inv = 1.f / den;
  const int n4 = D / 4;
  if (lane < n4) {
    const size_t off = static_cast<size_t>(row) * n4 + lane;
    const float4 a = reinterpret_cast<const float4 *>(o_a)[off];
    const float4 bb = reinterpret_cast<const float4 *>(o_b)[off];
    const float4 c = reinterpret_cast<const float4 *>(o_c)[off];
    float4 o;
    o.x = (wa * a.x + wb * bb.x - wc * c.x) * inv;
    o.y = (wa * a.y + wb * bb.y - wc * c.y) * inv;
    o.z = (wa * a.z + wb * bb.z - wc * c.z) * inv;
    o.w = (wa * a.w + wb * bb.w - wc * c.w) * inv;
    if (out_f32) {
      reinterpret_cast<float4 *>(out)[off] = o;
    } else {
      __nv_bfloat162 lo = __floats2bfloat162_rn(o.x, o.y), hi = __floats2bfloat162_rn(o.z, o.w);
      uint2 packed;
      packed.x = *reinterpret_cast<uint32_t *>(&lo);
      packed.y = *reinterpret_cast<uint32_t *>(&hi);
      reinterpret_cast<uint2 *>(out)[off] = packed;
    }
  }
  if (lane == 0 && lse) lse[li] = M + logf(den);
}

}  // namespace

cudaError_t launch_three_pass_merge(const float *o_a, const float *o_b, const float *o_c,
                                    const float *l_a, const float *l_b, const float *l_c,
                                    void *out, float *lse, int out_f32, int B, int Hq, int L,
                                    int D, cudaStream_t stream) {
  const long long rows = static_cast<long long>(B) * L * Hq;
  const long long blocks = (rows + kMergeWarps - 1) / kMergeWarps;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  three_pass_merge_kernel<<<static_cast<unsigned>(blocks), kMergeWarps * 32, 0, stream>>>(
      o_a, o_b, o_c, l_a, l_b, l_c, out, lse, out_f32, B, Hq, L, D);
  return cudaGetLastError();
}

}  // namespace jl
