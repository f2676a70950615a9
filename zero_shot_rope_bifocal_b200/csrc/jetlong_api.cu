// jetlong_api.cu -- the C ABI declared in include/jetlong.h: argument
// validation, workspace carving, and the launch sequence of each call.
//
// Every check runs on the host before the first CUDA call, so an invalid call
// returns its status without touching the device (and works on a machine with
// no GPU at all).
#include <algorithm>
#include <cmath>
#include <mutex>

#include "../../include/jetlong.h"
#include "jl_common.cuh"
#include "sm100_ptx.cuh"

namespace jl {

// Kernel-side error word (timeouts of bounded waits).  Kernels receive its
// device address; host code reaches it through cudaGetSymbolAddress.
__device__ unsigned int g_device_error;

std::atomic<unsigned> g_state_epoch{0};

void reset_noalloc_cache();  // defined with the jetlong_decode_noalloc buffer below

namespace {

constexpr size_t kAlign = 256;
constexpr long long kMaxGridYZ = 65535;  // CUDA's limit on gridDim.y and gridDim.z

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// One thread waits on an mbarrier that never completes, bounded by limit_ns,
// and records the timeout the way the attention kernels do.
__global__ void wait_timeout_check_kernel(unsigned int *dev_error, unsigned long long limit_ns) {
  __shared__ __align__(8) unsigned long long barrier_word;
  const uint32_t bar = smem_u32(&barrier_word);
  mbar_init(bar, 1);
  fence_mbar_init();
  if (!mbar_wait_bounded(bar, 0u, limit_ns)) atomicOr(dev_error, kDevTimeout);
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct DeviceState {
  bool checked = false;
  bool is_sm100 = false;
  unsigned int *err = nullptr;
};

constexpr int kMaxDevices = 64;
std::mutex g_mu;
DeviceState g_dev[kMaxDevices];

// Checks the current device once (compute capability 10.x) and fetches the
// device address of the error word for it.
int current_device(DeviceState **out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return JL_ERR_NO_DEVICE;
  }
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceState &st = g_dev[dev];
  if (!st.checked) {
    int major = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) {
      cudaGetLastError();
      return JL_ERR_NO_DEVICE;
    }
    st.is_sm100 = (major == 10);
    if (st.is_sm100) {
      void *p = nullptr;
      if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) {
        cudaGetLastError();
        return JL_ERR_CUDA;
      }
      st.err = static_cast<unsigned int *>(p);
    }
    st.checked = true;
  }
  if (!st.is_sm100) return JL_ERR_NO_DEVICE;
  *out = &st;
  return JL_OK;
}

int check_common(int B, int Hq, int Hkv, int L, int D) {
  if (B < 1 || Hq < 1 || Hkv < 1 || L < 1) return JL_ERR_SHAPE;
  if (Hq % Hkv != 0) return JL_ERR_SHAPE;
  if (D != 64 && D != 128) return JL_ERR_UNSUPPORTED;
  // Sizes must keep every element index inside 2^31 tokens x heads x D math.
  if (static_cast<long long>(B) * L * Hq > (1ll << 31)) return JL_ERR_SHAPE;
  return JL_OK;
}

int check_method(int w_pretrained, int w0, float theta) {
  if (w_pretrained < 1 || w0 < 0) return JL_ERR_SHAPE;
  if (!(theta > 0.f) || theta != theta) return JL_ERR_SHAPE;
  return JL_OK;
}

// Ramp bounds of the frequency-interpolation remote map: finite, beta > alpha.
int check_ramp(float alpha, float beta) {
  if (!std::isfinite(alpha) || !std::isfinite(beta) || !(beta > alpha)) return JL_ERR_SHAPE;
  return JL_OK;
}

// The key operands of a prefill: k_true, k_remote, v (FP16 [B, Hkv, L, D]).
// The queries need none: the attention kernel rotates them as it loads them.
size_t prefill_ws_bytes(int B, int /*Hq*/, int Hkv, int L, int D) {
  const size_t k = static_cast<size_t>(B) * Hkv * L * D * 2;
  return 3 * align_up(k);
}

// Three-pass workspace: the prefill operands, then O_A, O_B, O_C (fp32
// [B, L, Hq, D]) and lse_A, lse_B, lse_C (fp32 [B, Hq, L]).
size_t three_pass_ws_bytes(int B, int Hq, int Hkv, int L, int D) {
  const size_t o = align_up(static_cast<size_t>(B) * L * Hq * D * sizeof(float));
  const size_t l = align_up(static_cast<size_t>(B) * Hq * L * sizeof(float));
  return prefill_ws_bytes(B, Hq, Hkv, L, D) + 3 * o + 3 * l;
}

size_t decode_ws_bytes(int B, int Hq, int Hkv, int L, int D) {
  int ns = 0, ch = 0;
  decode_plan(B, Hkv, L, &ns, &ch);
  return align_up(static_cast<size_t>(B) * Hq * ns * (D + 2) * sizeof(float));
}

}  // namespace
}  // namespace jl

using namespace jl;

extern "C" {

const char *jetlong_status_string(int s) {
  switch (s) {
    case JL_OK: return "JL_OK";
    case JL_ERR_NULL: return "JL_ERR_NULL: a required pointer is NULL";
    case JL_ERR_SHAPE: return "JL_ERR_SHAPE: a size is out of range or inconsistent";
    case JL_ERR_UNSUPPORTED: return "JL_ERR_UNSUPPORTED: configuration not implemented";
    case JL_ERR_ALIGN: return "JL_ERR_ALIGN: a pointer is not 16-byte aligned";
    case JL_ERR_WORKSPACE: return "JL_ERR_WORKSPACE: workspace missing or too small";
    case JL_ERR_CUDA: return "JL_ERR_CUDA: a CUDA call or launch failed";
    case JL_ERR_DEVICE_TIMEOUT: return "JL_ERR_DEVICE_TIMEOUT: a bounded in-kernel wait expired";
    case JL_ERR_NO_DEVICE: return "JL_ERR_NO_DEVICE: no sm_100 device is current";
    case JL_ERR_RANGE: return "JL_ERR_RANGE: an input value exceeds the FP16 operand range";
    default: return "unknown jl_status";
  }
}

const char *jetlong_version(void) { return "0.1.0"; }

void jetlong_shutdown(void) {
  {
    std::lock_guard<std::mutex> lk(g_mu);
    for (DeviceState &st : g_dev) st = DeviceState{};
  }
  reset_noalloc_cache();
  g_state_epoch.fetch_add(1, std::memory_order_acq_rel);
}

int jetlong_group_size(int L, int w_pretrained) {
  if (L < 1 || w_pretrained < 1) return JL_ERR_SHAPE;
  return group_size(L, w_pretrained);
}

size_t jetlong_prefill_workspace_size(int B, int Hq, int Hkv, int L, int D) {
  if (check_common(B, Hq, Hkv, L, D) != JL_OK) return 0;
  return prefill_ws_bytes(B, Hq, Hkv, L, D);
}

}  // extern "C"

namespace {

// Which buffers a prefill entry point reads or writes.
enum PrefillStage : int { kStageRotate = 1, kStageAttend = 2, kStageBoth = 3 };

// Validation shared by the prefill entry points.  A stage's pointers must be
// non-NULL and aligned; pointers of the other stage must be NULL and are
// never handed to a kernel.
int prepare_prefill(int stage, const void *q, const void *k, const void *v, void *out, float *lse,
                    int B, int Hq, int Hkv, int L, int D, int w_pretrained, int w0,
                    float rope_theta, int out_dtype, void *k_cache_out, int k_cache_capacity,
                    void *workspace, size_t workspace_bytes, PrefillArgs *a,
                    bool three_pass = false) {
  const bool rot = stage & kStageRotate, att = stage & kStageAttend;
  if (rot && (!k || !v)) return JL_ERR_NULL;
  if (att && (!q || !out)) return JL_ERR_NULL;
  int st = check_common(B, Hq, Hkv, L, D);
  if (st != JL_OK) return st;
  // grids: (positions, batch) for the operand pass, (query tiles, KV heads x
  // head pairs, batch) for the attention kernel
  if (B > kMaxGridYZ || static_cast<long long>(Hkv) * ((Hq / Hkv + 1) / 2) > kMaxGridYZ)
    return JL_ERR_SHAPE;
  if ((st = check_method(w_pretrained, w0, rope_theta)) != JL_OK) return st;
  if (att && out_dtype != JL_BF16 && out_dtype != JL_F32) return JL_ERR_UNSUPPORTED;
  if (rot && k_cache_out && k_cache_capacity < L) return JL_ERR_SHAPE;
  if (rot && (!aligned16(k) || !aligned16(v) || (k_cache_out && !aligned16(k_cache_out))))
    return JL_ERR_ALIGN;
  if (att && (!aligned16(q) || !aligned16(out) || (lse && !aligned16(lse)))) return JL_ERR_ALIGN;
  const size_t need = three_pass ? three_pass_ws_bytes(B, Hq, Hkv, L, D)
                                 : prefill_ws_bytes(B, Hq, Hkv, L, D);
  if (!workspace || workspace_bytes < need) return JL_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(workspace) % kAlign) return JL_ERR_ALIGN;

  DeviceState *dev = nullptr;
  if ((st = current_device(&dev)) != JL_OK) return st;

  *a = PrefillArgs{};
  a->q = att ? static_cast<const __nv_bfloat16 *>(q) : nullptr;
  a->k = rot ? static_cast<const __nv_bfloat16 *>(k) : nullptr;
  a->v = rot ? static_cast<const __nv_bfloat16 *>(v) : nullptr;
  a->out = att ? out : nullptr;
  a->lse = att ? lse : nullptr;
  a->out_f32 = out_dtype == JL_F32;
  a->k_cache_out = rot ? static_cast<__nv_bfloat16 *>(k_cache_out) : nullptr;
  a->k_cache_capacity = a->k_cache_out ? k_cache_capacity : 0;
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  const size_t kb = align_up(static_cast<size_t>(B) * Hkv * L * D * 2);
  a->k_true = reinterpret_cast<__half *>(ws);
  a->k_remote = reinterpret_cast<__half *>(ws + kb);
  a->v_op = reinterpret_cast<__half *>(ws + 2 * kb);
  a->B = B;
  a->Hq = Hq;
  a->Hkv = Hkv;
  a->L = L;
  a->q_off = 0;
  a->Lq = L;
  a->D = D;
  a->w_pretrained = w_pretrained;
  a->w0 = w0;
  a->G = group_size(L, w_pretrained);
  a->theta = rope_theta;
  a->dev_error = dev->err;
  return JL_OK;
}

}  // namespace

extern "C" {

int jetlong_prefill(const void *q, const void *k, const void *v, void *out, float *lse, int B,
                    int Hq, int Hkv, int L, int D, int w_pretrained, int w0, float rope_theta,
                    int out_dtype, void *k_cache_out, int k_cache_capacity, void *workspace,
                    size_t workspace_bytes, jl_stream_t stream) {
  PrefillArgs a;
  const int st = prepare_prefill(kStageBoth, q, k, v, out, lse, B, Hq, Hkv, L, D, w_pretrained,
                                 w0, rope_theta, out_dtype, k_cache_out, k_cache_capacity,
                                 workspace, workspace_bytes, &a);
  if (st != JL_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (launch_rope_kv(a, s) != cudaSuccess) return JL_ERR_CUDA;
  if (launch_prefill_attention(a, s) != cudaSuccess) return JL_ERR_CUDA;
  return JL_OK;
}

int jetlong_prefill_interp(const void *q, const void *k, const void *v, void *out, float *lse,
                           int B, int Hq, int Hkv, int L, int D, int w_pretrained, int w0,
                           float rope_theta, float ramp_alpha, float ramp_beta, int out_dtype,
                           void *k_cache_out, int k_cache_capacity, void *workspace,
                           size_t workspace_bytes, jl_stream_t stream) {
  if (check_ramp(ramp_alpha, ramp_beta) != JL_OK) return JL_ERR_SHAPE;
  PrefillArgs a;
  const int st = prepare_prefill(kStageBoth, q, k, v, out, lse, B, Hq, Hkv, L, D, w_pretrained,
                                 w0, rope_theta, out_dtype, k_cache_out, k_cache_capacity,
                                 workspace, workspace_bytes, &a);
  if (st != JL_OK) return st;
  a.interp = 1;
  a.ramp_alpha = ramp_alpha;
  a.ramp_beta = ramp_beta;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (launch_rope_kv(a, s) != cudaSuccess) return JL_ERR_CUDA;
  if (launch_prefill_attention(a, s) != cudaSuccess) return JL_ERR_CUDA;
  return JL_OK;
}

int jetlong_prefill_rotate(const void *k, const void *v, int B, int Hkv, int L, int D,
                           int w_pretrained, float rope_theta, void *k_cache_out,
                           int k_cache_capacity, void *workspace, size_t workspace_bytes,
                           jl_stream_t stream) {
  PrefillArgs a;
  const int st = prepare_prefill(kStageRotate, nullptr, k, v, nullptr, nullptr, B, Hkv, Hkv, L, D,
                                 w_pretrained, 0, rope_theta, JL_BF16, k_cache_out,
                                 k_cache_capacity, workspace, workspace_bytes, &a);
  if (st != JL_OK) return st;
  if (launch_rope_kv(a, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return JL_ERR_CUDA;
  return JL_OK;
}

int jetlong_prefill_attend(const void *q, void *out, float *lse, int B, int Hq, int Hkv, int L,
                           int D, int w_pretrained, int w0, float rope_theta, int out_dtype,
                           const void *workspace, size_t workspace_bytes, jl_stream_t stream) {
  PrefillArgs a;
  const int st = prepare_prefill(kStageAttend, q, nullptr, nullptr, out, lse, B, Hq, Hkv, L, D,
                                 w_pretrained, w0, rope_theta, out_dtype, nullptr, 0,
                                 const_cast<void *>(workspace), workspace_bytes, &a);
  if (st != JL_OK) return st;
  if (launch_prefill_attention(a, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return JL_ERR_CUDA;
  return JL_OK;
}

size_t jetlong_prefill_three_pass_workspace_size(int B, int Hq, int Hkv, int L, int D) {
  if (check_common(B, Hq, Hkv, L, D) != JL_OK) return 0;
  return three_pass_ws_bytes(B, Hq, Hkv, L, D);
}

int jetlong_prefill_three_pass(const void *q, const void *k, const void *v, void *out, float *lse,
                               int B, int Hq, int Hkv, int L, int D, int w_pretrained, int w0,
                               float rope_theta, int out_dtype, void *workspace,
                               size_t workspace_bytes, jl_stream_t stream) {
  PrefillArgs a;
  const int st = prepare_prefill(kStageBoth, q, k, v, out, lse, B, Hq, Hkv, L, D, w_pretrained,
                                 w0, rope_theta, out_dtype, nullptr, 0, workspace, workspace_bytes,
                                 &a, /*three_pass=*/true);
  if (st != JL_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t *ws = static_cast<uint8_t *>(workspace) + prefill_ws_bytes(B, Hq, Hkv, L, D);
  const size_t ob = align_up(static_cast<size_t>(B) * L * Hq * D * sizeof(float));
  const size_t lb = align_up(static_cast<size_t>(B) * Hq * L * sizeof(float));
  float *o_pass[3], *l_pass[3];
  for (int i = 0; i < 3; ++i) {
    o_pass[i] = reinterpret_cast<float *>(ws + i * ob);
    l_pass[i] = reinterpret_cast<float *>(ws + 3 * ob + i * lb);
  }
  if (launch_rope_kv(a, s) != cudaSuccess) return JL_ERR_CUDA;
  const PrefillPass passes[3] = {kPassRemoteCausal, kPassLocalBand, kPassRemoteBand};
  for (int i = 0; i < 3; ++i) {
    PrefillArgs p = a;
    p.pass = passes[i];
    p.out = o_pass[i];
    p.lse = l_pass[i];
    p.out_f32 = 1;
    if (launch_prefill_attention(p, s) != cudaSuccess) return JL_ERR_CUDA;
  }
  if (launch_three_pass_merge(o_pass[0], o_pass[1], o_pass[2], l_pass[0], l_pass[1], l_pass[2],
                              out, lse, out_dtype == JL_F32, B, Hq, L, D, s) != cudaSuccess)
    return JL_ERR_CUDA;
  return JL_OK;
}

size_t jetlong_decode_workspace_size(int B, int Hq, int Hkv, int L, int D) {
  if (check_common(B, Hq, Hkv, L, D) != JL_OK) return 0;
  return decode_ws_bytes(B, Hq, Hkv, L, D);
}

}  // extern "C"

namespace {

// Queries at positions q_pos0 .. q_pos0 + nq - 1 (per batch entry) against the
// true-position cache, each over keys [0, its position], with one G from the
// longest range L = q_pos0 + nq: a decode step (nq = 1) or a prefill chunk.
// The decode kernels' turn fractions (theta_i / (2 pi) as 64-bit binary
// fractions) for the call's theta, map and length.
void fill_decode_turns(DecodeArgs *a) {
  const double turns_q64 = 0.15915494309189533577 * 18446744073709551616.0;  // 2^64 / (2 pi)
  const double log_theta = std::log(static_cast<double>(a->theta));
  for (int i = 0; i < a->D / 2; ++i) {
    const double f = std::exp(-2.0 * static_cast<double>(i) / static_cast<double>(a->D) * log_theta);
    const double factor =
        a->interp ? interp_factor(f, a->L, a->w_pretrained, a->ramp_alpha, a->ramp_beta) : 1.0;
    a->omega_qt[i] = static_cast<uint64_t>(std::llround(f * turns_q64));  // < 2^62
    a->omega_qr[i] = static_cast<uint64_t>(std::llround(f * factor * turns_q64));
    // (theta' - theta) / (2 pi) lies in (-1/(2 pi), 0]: inside int64 once scaled
    a->omega_corr[i] = a->interp ? static_cast<uint64_t>(std::llround(f * (factor - 1.0) * turns_q64))
                                 : a->omega_qt[i];
  }
}

// Every host check of such a call except the workspace's; sets *L_out to the
// key range q_pos0 + nq.  Makes no CUDA call.
int check_cache_call(const void *q, const void *k_cache, const void *v_cache, const void *out,
                     const float *lse, int B, int Hq, int Hkv, int nq, int q_pos0, int Lcap, int D,
                     int w_pretrained, int w0, float rope_theta, int out_dtype, int interp,
                     float ramp_alpha, float ramp_beta, const void *k_remote, int *L_out) {
  if (!q || !k_cache || !v_cache || !out) return JL_ERR_NULL;
  if (k_remote && !aligned16(k_remote)) return JL_ERR_ALIGN;
  if (interp && check_ramp(ramp_alpha, ramp_beta) != JL_OK) return JL_ERR_SHAPE;
  if (nq < 1 || q_pos0 < 0) return JL_ERR_SHAPE;
  const long long L_ll = static_cast<long long>(q_pos0) + nq;
  if (L_ll > (1ll << 31) - 1) return JL_ERR_SHAPE;
  const int L = static_cast<int>(L_ll);
  int st = check_common(B, Hq, Hkv, L, D);
  if (st != JL_OK) return st;
  if (static_cast<long long>(B) * nq > 65535) return JL_ERR_SHAPE;  // grid z of the split kernel
  if (static_cast<long long>(B) * nq * Hq * L > (1ll << 40)) return JL_ERR_SHAPE;
  if (Lcap < L) return JL_ERR_SHAPE;
  if (!decode_supports_group(Hq / Hkv)) return JL_ERR_UNSUPPORTED;
  if ((Hkv + 7) / 8 > kMaxGridYZ) return JL_ERR_SHAPE;  // grid y: groups of 8 KV heads
  if ((st = check_method(w_pretrained, w0, rope_theta)) != JL_OK) return st;
  if (out_dtype != JL_BF16 && out_dtype != JL_F32) return JL_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) ||
      (lse && !aligned16(lse)))
    return JL_ERR_ALIGN;
  *L_out = L;
  return JL_OK;
}

int cache_attention(const void *q, const void *k_cache, const void *v_cache, void *out, float *lse,
                    int B, int Hq, int Hkv, int nq, int q_pos0, int Lcap, int D, int w_pretrained,
                    int w0, float rope_theta, int out_dtype, void *workspace,
                    size_t workspace_bytes, jl_stream_t stream, int interp = 0,
                    float ramp_alpha = 0.f, float ramp_beta = 0.f,
                    const void *k_remote = nullptr) {
  int L = 0;
  int st = check_cache_call(q, k_cache, v_cache, out, lse, B, Hq, Hkv, nq, q_pos0, Lcap, D,
                            w_pretrained, w0, rope_theta, out_dtype, interp, ramp_alpha,
                            ramp_beta, k_remote, &L);
  if (st != JL_OK) return st;
  const size_t need = decode_ws_bytes(B * nq, Hq, Hkv, L, D);
  if (!workspace || workspace_bytes < need) return JL_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(workspace) % kAlign) return JL_ERR_ALIGN;

  DeviceState *dev = nullptr;
  if ((st = current_device(&dev)) != JL_OK) return st;

  DecodeArgs a{};
  a.q = static_cast<const __nv_bfloat16 *>(q);
  a.k_cache = static_cast<const __nv_bfloat16 *>(k_cache);
  a.v_cache = static_cast<const __nv_bfloat16 *>(v_cache);
  a.k_remote = static_cast<const __half *>(k_remote);
  a.out = out;
  a.lse = lse;
  a.out_f32 = out_dtype == JL_F32;
  a.partial = static_cast<float *>(workspace);
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.L = L;
  a.Lcap = Lcap;
  a.D = D;
  a.w_pretrained = w_pretrained;
  a.w0 = w0;
  a.G = group_size(L, w_pretrained);
  a.gdiv = make_group_divider(a.G);
  a.theta = rope_theta;
  a.nq = nq;
  a.q_pos0 = q_pos0;
  a.interp = interp;
  a.ramp_alpha = ramp_alpha;
  a.ramp_beta = ramp_beta;
  decode_plan(B * nq, Hkv, L, &a.n_split, &a.chunk);
  fill_decode_turns(&a);
  a.dev_error = dev->err;
  if (launch_decode(a, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return JL_ERR_CUDA;
  return JL_OK;
}

// A chunk of at least JL_CHUNK_TENSOR_MIN queries (include/jetlong.h) runs on
// the tensor-core prefill kernel (key operands converted once, 128-row query
// tiles, the keys split when the tiles are few); shorter chunks run on the
// decode kernels, one split-KV problem per query, whose cost is n passes over
// the cache: on a 128K cache the two meet at about 5 queries.
constexpr int kChunkTensorMin = JL_CHUNK_TENSOR_MIN;

// Key split of the tensor-core chunk path: a chunk of few query tiles would
// leave most SMs idle (one CTA per SM, each walking all of its tile's key
// tiles), so each tile's visits are split into ranges, one CTA each, up to one
// wave of 148 CTAs, and merged by log-sum-exp.  Every split keeps at least one
// visit: the first query tile visits at least (its last position) / 128 + 1
// key tiles under the fused rule.
int chunk_split_count(int B, int Hq, int Hkv, int P0, int n) {
  constexpr int kSms = 148;
  const long long ctas = static_cast<long long>((n + 127) / 128) * Hkv * ((Hq / Hkv + 1) / 2) * B;
  if (ctas * 2 > kSms) return 1;
  int ns = static_cast<int>(kSms / ctas);
  ns = std::min(ns, (std::min(P0 + 128, P0 + n) - 1) / 128 + 1);
  ns = std::min(ns, static_cast<int>(kMaxGridYZ / B));
  return std::max(ns, 1);
}

// Workspace of the tensor-core chunk path: the FP16 key operands, cached
// keys in both forms and values [B, Hkv, P0 + n, D] (the kernel rotates the
// chunk's queries as it loads them), then the split records
// [B, n, Hq, n_split, D + 2] fp32 when the keys are split.
size_t chunk_tensor_ws_bytes(int B, int Hq, int Hkv, int P0, int n, int D) {
  const size_t k = align_up(static_cast<size_t>(B) * Hkv * (static_cast<size_t>(P0) + n) * D * 2);
  const int ns = chunk_split_count(B, Hq, Hkv, P0, n);
  const size_t rec = ns > 1 ? align_up(static_cast<size_t>(B) * n * Hq * ns * (D + 2) * 4) : 0;
  return 3 * k + rec;
}

size_t chunk_ws_bytes(int B, int Hq, int Hkv, int P0, int n, int D) {
  return n >= kChunkTensorMin ? chunk_tensor_ws_bytes(B, Hq, Hkv, P0, n, D)
                              : decode_ws_bytes(B * n, Hq, Hkv, P0 + n, D);
}

// A prefill chunk on the tensor-core prefill kernel: the chunk's queries
// (positions P0 .. P0 + n - 1) against keys [0, P0 + n) of the true-position
// cache, with the same score rule and one G from P0 + n.
int chunk_tensor(const void *q, const void *k_cache, const void *v_cache, void *out, float *lse,
                 int B, int Hq, int Hkv, int P0, int n, int Lcap, int D, int w_pretrained,
                 int w0, float rope_theta, int out_dtype, void *workspace,
                 size_t workspace_bytes, jl_stream_t stream, int interp, float ramp_alpha,
                 float ramp_beta) {
  int L = 0;
  int st = check_cache_call(q, k_cache, v_cache, out, lse, B, Hq, Hkv, n, P0, Lcap, D,
                            w_pretrained, w0, rope_theta, out_dtype, interp, ramp_alpha,
                            ramp_beta, nullptr, &L);
  if (st != JL_OK) return st;
  // grids: (query tiles, KV heads x head pairs, batch) and (positions, batch)
  if (B > kMaxGridYZ || static_cast<long long>(Hkv) * ((Hq / Hkv + 1) / 2) > kMaxGridYZ)
    return JL_ERR_SHAPE;
  const size_t need = chunk_tensor_ws_bytes(B, Hq, Hkv, P0, n, D);
  if (!workspace || workspace_bytes < need) return JL_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(workspace) % kAlign) return JL_ERR_ALIGN;
  DeviceState *dev = nullptr;
  if ((st = current_device(&dev)) != JL_OK) return st;

  PrefillArgs a{};
  a.q = static_cast<const __nv_bfloat16 *>(q);
  a.out = out;
  a.lse = lse;
  a.out_f32 = out_dtype == JL_F32;
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  const size_t kb = align_up(static_cast<size_t>(B) * Hkv * L * D * 2);
  a.k_true = reinterpret_cast<__half *>(ws);
  a.k_remote = reinterpret_cast<__half *>(ws + kb);
  a.v_op = reinterpret_cast<__half *>(ws + 2 * kb);
  a.n_split = chunk_split_count(B, Hq, Hkv, P0, n);
  a.partial = a.n_split > 1 ? reinterpret_cast<float *>(ws + 3 * kb) : nullptr;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.L = L;
  a.D = D;
  a.w_pretrained = w_pretrained;
  a.w0 = w0;
  a.G = group_size(L, w_pretrained);
  a.theta = rope_theta;
  a.q_off = P0;
  a.Lq = n;
  a.k_cache_in = static_cast<const __nv_bfloat16 *>(k_cache);
  a.v_cache_in = static_cast<const __nv_bfloat16 *>(v_cache);
  a.cache_cap = Lcap;
  a.interp = interp;
  a.ramp_alpha = ramp_alpha;
  a.ramp_beta = ramp_beta;
  a.dev_error = dev->err;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (launch_chunk_operands(a, s) != cudaSuccess) return JL_ERR_CUDA;
  if (launch_prefill_attention(a, s) != cudaSuccess) return JL_ERR_CUDA;
  return JL_OK;
}

}  // namespace

extern "C" {

int jetlong_decode(const void *q, const void *k_cache, const void *v_cache, void *out, float *lse,
                   int B, int Hq, int Hkv, int L, int Lcap, int D, int w_pretrained, int w0,
                   float rope_theta, int out_dtype, void *workspace, size_t workspace_bytes,
                   jl_stream_t stream) {
  if (L < 1) return JL_ERR_SHAPE;
  return cache_attention(q, k_cache, v_cache, out, lse, B, Hq, Hkv, 1, L - 1, Lcap, D,
                         w_pretrained, w0, rope_theta, out_dtype, workspace, workspace_bytes,
                         stream);
}

size_t jetlong_prefill_chunk_workspace_size(int B, int Hq, int Hkv, int P0, int n, int D) {
  if (n < 1 || P0 < 0 || static_cast<long long>(P0) + n > (1ll << 31) - 1) return 0;
  if (check_common(B, Hq, Hkv, P0 + n, D) != JL_OK) return 0;
  if (static_cast<long long>(B) * n > 65535) return 0;
  return chunk_ws_bytes(B, Hq, Hkv, P0, n, D);
}

int jetlong_prefill_chunk(const void *q, const void *k_cache, const void *v_cache, void *out,
                          float *lse, int B, int Hq, int Hkv, int P0, int n, int Lcap, int D,
                          int w_pretrained, int w0, float rope_theta, int out_dtype,
                          void *workspace, size_t workspace_bytes, jl_stream_t stream) {
  if (n >= kChunkTensorMin)
    return chunk_tensor(q, k_cache, v_cache, out, lse, B, Hq, Hkv, P0, n, Lcap, D, w_pretrained,
                        w0, rope_theta, out_dtype, workspace, workspace_bytes, stream, 0, 0.f,
                        0.f);
  return cache_attention(q, k_cache, v_cache, out, lse, B, Hq, Hkv, n, P0, Lcap, D,
                         w_pretrained, w0, rope_theta, out_dtype, workspace, workspace_bytes,
                         stream);
}

int jetlong_decode_interp(const void *q, const void *k_cache, const void *v_cache, void *out,
                          float *lse, int B, int Hq, int Hkv, int L, int Lcap, int D,
                          int w_pretrained, int w0, float rope_theta, float ramp_alpha,
                          float ramp_beta, int out_dtype, void *workspace, size_t workspace_bytes,
                          jl_stream_t stream) {
  if (L < 1) return JL_ERR_SHAPE;
  return cache_attention(q, k_cache, v_cache, out, lse, B, Hq, Hkv, 1, L - 1, Lcap, D,
                         w_pretrained, w0, rope_theta, out_dtype, workspace, workspace_bytes,
                         stream, 1, ramp_alpha, ramp_beta);
}

int jetlong_prefill_chunk_interp(const void *q, const void *k_cache, const void *v_cache,
                                 void *out, float *lse, int B, int Hq, int Hkv, int P0, int n,
                                 int Lcap, int D, int w_pretrained, int w0, float rope_theta,
                                 float ramp_alpha, float ramp_beta, int out_dtype, void *workspace,
                                 size_t workspace_bytes, jl_stream_t stream) {
  if (n >= kChunkTensorMin)
    return chunk_tensor(q, k_cache, v_cache, out, lse, B, Hq, Hkv, P0, n, Lcap, D, w_pretrained,
                        w0, rope_theta, out_dtype, workspace, workspace_bytes, stream, 1,
                        ramp_alpha, ramp_beta);
  return cache_attention(q, k_cache, v_cache, out, lse, B, Hq, Hkv, n, P0, Lcap, D,
                         w_pretrained, w0, rope_theta, out_dtype, workspace, workspace_bytes,
                         stream, 1, ramp_alpha, ramp_beta);
}

int jetlong_remote_cache(const void *k_cache, void *k_remote, int B, int Lcap, int Hkv, int D,
                         int j0, int j1, int L, int w_pretrained, float rope_theta,
                         jl_stream_t stream) {
  if (!k_cache || !k_remote) return JL_ERR_NULL;
  if (B < 1 || B > 65535 || Hkv < 1 || L < 1 || Lcap < L) return JL_ERR_SHAPE;
  if (j0 < 0 || j1 < j0 || j1 > L) return JL_ERR_SHAPE;
  if (D != 64 && D != 128) return JL_ERR_UNSUPPORTED;
  int st = check_method(w_pretrained, 0, rope_theta);
  if (st != JL_OK) return st;
  if (!aligned16(k_cache) || !aligned16(k_remote)) return JL_ERR_ALIGN;
  if (j0 == j1) return JL_OK;
  DeviceState *dev = nullptr;
  if ((st = current_device(&dev)) != JL_OK) return st;
  if (launch_remote_cache(static_cast<const __nv_bfloat16 *>(k_cache), static_cast<__half *>(k_remote),
                          B, Lcap, Hkv, D, j0, j1, group_size(L, w_pretrained), rope_theta,
                          reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return JL_ERR_CUDA;
  return JL_OK;
}

int jetlong_decode_two_form(const void *q, const void *k_cache, const void *k_remote,
                            const void *v_cache, void *out, float *lse, int B, int Hq, int Hkv,
                            int L, int Lcap, int D, int w_pretrained, int w0, float rope_theta,
                            int out_dtype, void *workspace, size_t workspace_bytes,
                            jl_stream_t stream) {
  if (!k_remote) return JL_ERR_NULL;
  if (L < 1) return JL_ERR_SHAPE;
  return cache_attention(q, k_cache, v_cache, out, lse, B, Hq, Hkv, 1, L - 1, Lcap, D,
                         w_pretrained, w0, rope_theta, out_dtype, workspace, workspace_bytes,
                         stream, 0, 0.f, 0.f, k_remote);
}

int jetlong_rope_cache(const void *k, void *k_cache, int B, int n, int Hkv, int D, int pos0,
                       int Lcap, float rope_theta, jl_stream_t stream) {
  if (!k || !k_cache) return JL_ERR_NULL;
  if (B < 1 || B > kMaxGridYZ || n < 1 || Hkv < 1 || pos0 < 0 || Lcap < 1) return JL_ERR_SHAPE;
  if (static_cast<long long>(pos0) + n > Lcap) return JL_ERR_SHAPE;
  if (D != 64 && D != 128) return JL_ERR_UNSUPPORTED;
  if (!(rope_theta > 0.f)) return JL_ERR_SHAPE;
  if (!aligned16(k) || !aligned16(k_cache)) return JL_ERR_ALIGN;
  DeviceState *dev = nullptr;
  int st = current_device(&dev);
  if (st != JL_OK) return st;
  if (launch_rope_cache(static_cast<const __nv_bfloat16 *>(k), static_cast<__nv_bfloat16 *>(k_cache),
                        B, n, Hkv, D, pos0, Lcap, rope_theta,
                        reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return JL_ERR_CUDA;
  return JL_OK;
}

int jetlong_check_device_timeout(int limit_ms, jl_stream_t stream) {
  if (limit_ms < 1 || limit_ms > 2000) return JL_ERR_SHAPE;
  DeviceState *dev = nullptr;
  const int st = current_device(&dev);
  if (st != JL_OK) return st;
  wait_timeout_check_kernel<<<1, 1, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      dev->err, static_cast<unsigned long long>(limit_ms) * 1000000ull);
  return cudaGetLastError() == cudaSuccess ? JL_OK : JL_ERR_CUDA;
}

int jetlong_device_status(jl_stream_t stream) {
  DeviceState *dev = nullptr;
  int st = current_device(&dev);
  if (st != JL_OK) return st;
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) {
    cudaGetLastError();
    return JL_ERR_CUDA;
  }
  unsigned int flag = 0;
  if (cudaMemcpyFromSymbol(&flag, g_device_error, sizeof(flag)) != cudaSuccess) return JL_ERR_CUDA;
  if (flag != kDevOk) {
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero)) != cudaSuccess) return JL_ERR_CUDA;
    return (flag & kDevTimeout) ? JL_ERR_DEVICE_TIMEOUT : JL_ERR_RANGE;
  }
  return JL_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Decode without any device allocation.
//
// Some callers cannot hand this library a workspace: their process forbids
// cudaMalloc outside start-up (a serving loop whose device memory is owned by
// one arena or caching allocator, or a latency-critical generation loop where
// an allocation would stall the device).  jetlong_decode_noalloc gives them
// the decode step with its split partials kept in a fixed buffer that lives in
// this library's device image instead.  Every GPU that loads the library holds
// this buffer until the process exits.
namespace jl {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;  // 8 MiB

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mu;
void *g_noalloc_ptr[kMaxDevices] = {};

// Device address of the scratch buffer on the current device.  The first call
// on a device looks it up (with that device current) and keeps it.
int noalloc_scratch(void **out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return JL_ERR_NO_DEVICE;
  }
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void *ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) {
      cudaGetLastError();
      return JL_ERR_CUDA;
    }
    g_noalloc_ptr[dev] = ptr;
  }
  *out = g_noalloc_ptr[dev];
  return JL_OK;
}

}  // namespace

void reset_noalloc_cache() {
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  for (void *&p : g_noalloc_ptr) p = nullptr;
}

}  // namespace jl

extern "C" int jetlong_decode_noalloc(const void *q, const void *k_cache, const void *v_cache,
                                      void *out, float *lse, int B, int Hq, int Hkv, int L,
                                      int Lcap, int D, int w_pretrained, int w0, float rope_theta,
                                      int out_dtype, jl_stream_t stream) {
  // Every argument check first, as for jetlong_decode: an invalid call
  // returns its status with no CUDA call.
  if (L < 1) return JL_ERR_SHAPE;
  int L_checked = 0;
  int st = check_cache_call(q, k_cache, v_cache, out, lse, B, Hq, Hkv, 1, L - 1, Lcap, D,
                            w_pretrained, w0, rope_theta, out_dtype, 0, 0.f, 0.f, nullptr,
                            &L_checked);
  if (st != JL_OK) return st;
  if (decode_ws_bytes(B, Hq, Hkv, L, D) > kNoAllocScratchBytes) return JL_ERR_WORKSPACE;
  // Then the device (an sm_100 one), and only then the buffer's address.
  DeviceState *dev = nullptr;
  if ((st = current_device(&dev)) != JL_OK) return st;
  void *scratch = nullptr;
  if ((st = noalloc_scratch(&scratch)) != JL_OK) return st;
  return jetlong_decode(q, k_cache, v_cache, out, lse, B, Hq, Hkv, L, Lcap, D, w_pretrained, w0,
                        rope_theta, out_dtype, scratch, kNoAllocScratchBytes, stream);
}
