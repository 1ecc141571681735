// zattn_api.cu -- the C ABI declared in include/zattn.h: argument
// validation, device checks and kernel launches.  No allocation, no
// synchronisation, no state kept between calls.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "zattn.h"

#include "schedule.h"
#include "zq_internal.h"

namespace {

constexpr int kVersion = 100;  // 0.1.0
constexpr uint64_t kTimeoutNs = 2000000000ull;  // bound on any single device-side wait
constexpr int64_t kMaxGroupedSlots = 65535;      // grouped quantiser: slots are grid.y

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Current device must be sm_100 (B200 class).  Returns the SM count through
// `num_sms` when non-null.
int check_device(int* num_sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ZQ_ERR_CUDA;
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return ZQ_ERR_CUDA;
  if (major != 10 || minor != 0) return ZQ_ERR_ARCH;
  if (num_sms &&
      cudaDeviceGetAttribute(num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return ZQ_ERR_CUDA;
  return ZQ_OK;
}

int validate_attn(const zq_attn_args* a) {
  if (!a) return ZQ_ERR_NULL;
  if (!a->q || !a->k || !a->v || !a->out) return ZQ_ERR_NULL;
  if (a->B <= 0 || a->Sq <= 0 || a->Sk <= 0 || a->Hq <= 0 || a->Hkv <= 0) return ZQ_ERR_SHAPE;
  if (a->Hq % a->Hkv != 0) return ZQ_ERR_SHAPE;
  if (!((a->d_qk == 128 && a->d_v == 128) || (a->d_qk == 192 && a->d_v == 128)))
    return ZQ_ERR_UNSUPPORTED;
  if (a->dtype != ZQ_DTYPE_BF16 && a->dtype != ZQ_DTYPE_FP8_E4M3) return ZQ_ERR_UNSUPPORTED;
  if (a->dtype == ZQ_DTYPE_FP8_E4M3) {
    if (a->softmax_mode != ZQ_SOFTMAX_EXACT && a->softmax_mode != ZQ_SOFTMAX_LEANP)
      return ZQ_ERR_UNSUPPORTED;
    if (a->block_scale != 0 && a->block_scale != 1) return ZQ_ERR_UNSUPPORTED;
    if (a->headroom_T < 0 || a->headroom_T > 8) return ZQ_ERR_UNSUPPORTED;
    if (a->descale_layout != ZQ_DESCALE_PER_TENSOR && a->descale_layout != ZQ_DESCALE_PER_KV_HEAD)
      return ZQ_ERR_UNSUPPORTED;
  }
  if (!(std::isfinite(a->softmax_scale))) return ZQ_ERR_SHAPE;
  // units = n_qtiles * B * Hq stay in int range, with room above the last
  // unit for the persistent CTAs' zigzag walk (it computes indices up to
  // two rounds of CTAs past the last unit); TMA element counts and strides
  const int64_t ntiles = (a->Sq + 127) / 128;
  if (ntiles * a->B * (int64_t)a->Hq > 0x7FFF0000ll) return ZQ_ERR_SHAPE;
  const int es = a->dtype == ZQ_DTYPE_BF16 ? 2 : 1;
  const int64_t qbytes = (int64_t)a->B * a->Sq * a->Hq * a->d_qk * es;
  const int64_t kbytes = (int64_t)a->B * a->Sk * a->Hkv * a->d_qk * es;
  if (qbytes >= (1ll << 40) || kbytes >= (1ll << 40)) return ZQ_ERR_SHAPE;
  if (!aligned16(a->q) || !aligned16(a->k) || !aligned16(a->v) || !aligned16(a->out) ||
      (a->lse && !aligned16(a->lse)))
    return ZQ_ERR_ALIGN;
  return ZQ_OK;
}

}  // namespace

extern "C" {

int zq_version(void) { return kVersion; }

const char* zq_status_string(int s) {
  switch (s) {
    case ZQ_OK: return "ok";
    case ZQ_ERR_NULL: return "a required pointer is NULL";
    case ZQ_ERR_SHAPE: return "invalid shape (size <= 0, Hq % Hkv != 0 or too large)";
    case ZQ_ERR_UNSUPPORTED: return "unsupported head dims, dtype, mode or option";
    case ZQ_ERR_ALIGN: return "pointer not 16-byte aligned";
    case ZQ_ERR_ARCH: return "current device is not sm_100 (B200)";
    case ZQ_ERR_CUDA: return "CUDA call failed";
    case ZQ_ERR_TIMEOUT: return "a device-side wait timed out";
    default: return "unknown status";
  }
}

// Launch description of a validated call (no device access).
static zq::AttnLaunch make_launch(const zq_attn_args* a) {
  zq::AttnLaunch L;
  L.q = a->q;
  L.k = a->k;
  L.v = a->v;
  L.dqk = a->d_qk;
  L.dv = a->d_v;
  L.dtype = a->dtype;
  L.mode = a->softmax_mode;
  L.block_scale = a->block_scale;
  L.p.out = a->out;
  L.p.lse = a->lse;
  L.p.q_descale = a->q_descale;
  L.p.k_descale = a->k_descale;
  L.p.v_descale = a->v_descale;
  L.p.descale_per_kv =
      a->dtype == ZQ_DTYPE_FP8_E4M3 && a->descale_layout == ZQ_DESCALE_PER_KV_HEAD ? 1 : 0;
  L.p.status = a->status;
  L.p.B = a->B;
  L.p.Sq = a->Sq;
  L.p.Sk = a->Sk;
  L.p.Hq = a->Hq;
  L.p.Hkv = a->Hkv;
  L.p.n_qtiles = (a->Sq + zq::kTile - 1) / zq::kTile;
  L.p.head_group = zq::choose_head_group(a->B, a->Hq, a->Hkv, a->Sq, a->Sk, a->d_qk, a->d_v,
                                         a->dtype == ZQ_DTYPE_FP8_E4M3 ? 1 : 2);
  L.p.causal = a->causal ? 1 : 0;
  L.p.headroom_T = a->dtype == ZQ_DTYPE_FP8_E4M3 ? a->headroom_T : 8;
  L.p.softmax_scale =
      a->softmax_scale > 0.0f ? a->softmax_scale : (float)(1.0 / std::sqrt((double)a->d_qk));
  L.p.timeout_ns = kTimeoutNs;
  L.p.dbg = nullptr;
  L.p.dbg_bh = 0;
  L.p.dbg_t = 0;
  L.p.dbg_flags = 0;
  return L;
}

static int attn_impl(const zq_attn_args* a, void* dbg, int dbg_bh, int dbg_t, int dbg_flags,
                     void* stream) {
  int rc = validate_attn(a);
  if (rc != ZQ_OK) return rc;
  rc = check_device(nullptr);
  if (rc != ZQ_OK) return rc;
  zq::AttnLaunch L = make_launch(a);
  L.p.dbg = dbg;
  L.p.dbg_bh = dbg_bh;
  L.p.dbg_t = dbg_t;
  L.p.dbg_flags = dbg_flags;
  cudaError_t e = zq::launch_attention(L, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? ZQ_OK : ZQ_ERR_CUDA;
}

int zq_attn_fwd_ex(const zq_attn_args* a, void* stream) {
  return attn_impl(a, nullptr, 0, 0, 0, stream);
}

int zq_attn_plan_launch(const zq_attn_args* a, int num_sms, zq_attn_plan* plan,
                        int32_t* unit_tile, int32_t* unit_bh, int32_t* unit_nkv,
                        int32_t* unit_cta, int32_t* unit_round) {
  if (!plan) return ZQ_ERR_NULL;
  int rc = validate_attn(a);
  if (rc != ZQ_OK) return rc;
  if (num_sms <= 0) {
    rc = check_device(&num_sms);
    if (rc != ZQ_OK) return rc;
  }
  const zq::AttnLaunch L = make_launch(a);
  const zq::AttnParams& p = L.p;
  // the kernel launch_attention picks: pairs of query tiles with 64-key
  // tiles (BF16, d = 128, more than 64 query tiles), else single query
  // tiles with 128-key tiles
  const bool pair = zq::use_pair_kernel(L.dtype, L.dqk, p.n_qtiles);
  const long long n_units = (long long)(pair ? zq::n_pairs_of(p.n_qtiles) : p.n_qtiles) * p.B * p.Hq;
  const long long grid = zq::grid_size(p.n_qtiles, n_units, num_sms);
  plan->n_units = n_units;
  plan->grid = grid;
  plan->persistent = zq::use_persistent(p.n_qtiles) ? 1 : 0;
  plan->head_group = p.head_group;
  plan->smem_bytes = pair ? zq::attn_pp_smem_bytes() : zq::attn_smem_bytes(a->dtype, a->d_qk);
  plan->threads = pair ? zq::attn_pp_threads() : zq::attn_threads();
  plan->rows_per_unit = pair ? 2 * zq::kTile : zq::kTile;
  plan->keys_per_tile = pair ? zq::kPairKeyTile : zq::kTile;
  if (!unit_tile && !unit_bh && !unit_nkv && !unit_cta && !unit_round) return ZQ_OK;
  for (long long u = 0; u < n_units; ++u) {
    int t, bh, nkv;
    if (pair) {
      const zq::PairUnit w = zq::pair_of(p, (int)u);
      t = w.tp, bh = w.bh, nkv = w.n_kv_max;
    } else {
      const zq::Unit w = zq::unit_of(p, (int)u);
      t = w.t, bh = w.bh, nkv = w.n_kv;
    }
    if (unit_tile) unit_tile[u] = t;
    if (unit_bh) unit_bh[u] = bh;
    if (unit_nkv) unit_nkv[u] = nkv;
  }
  if (unit_cta || unit_round) {
    // walk every CTA's sequence exactly as the kernel does
    for (long long c = 0; c < grid; ++c) {
      for (int k = 0;; ++k) {
        const long long u = zq::unit_at(k, (int)grid, (int)c);
        if (u >= n_units || (k > 0 && !plan->persistent)) break;
        if (unit_cta) unit_cta[u] = (int32_t)c;
        if (unit_round) unit_round[u] = k;
      }
    }
  }
  return ZQ_OK;
}

int zq_attn_fwd_debug(const zq_attn_args* a, void* dbg, int dbg_bh, int dbg_qtile, int flags,
                      void* stream) {
  if (!dbg) return ZQ_ERR_NULL;
  if (flags & ~1) return ZQ_ERR_UNSUPPORTED;
  return attn_impl(a, dbg, dbg_bh, dbg_qtile, flags, stream);
}

int zq_attn_fwd(const void* q, const void* k, const void* v, void* out, float* lse, int B,
                int Sq, int Sk, int Hq, int Hkv, int d_qk, int d_v, float softmax_scale,
                int causal, int dtype, const float* q_descale, const float* k_descale,
                const float* v_descale, void* stream) {
  zq_attn_args a;
  a.q = q;
  a.k = k;
  a.v = v;
  a.out = out;
  a.lse = lse;
  a.B = B;
  a.Sq = Sq;
  a.Sk = Sk;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.d_qk = d_qk;
  a.d_v = d_v;
  a.softmax_scale = softmax_scale;
  a.causal = causal;
  a.dtype = dtype;
  a.q_descale = q_descale;
  a.k_descale = k_descale;
  a.v_descale = v_descale;
  a.softmax_mode = ZQ_SOFTMAX_LEANP;
  a.block_scale = 1;
  a.headroom_T = 8;
  a.status = nullptr;
  a.descale_layout = ZQ_DESCALE_PER_TENSOR;
  return zq_attn_fwd_ex(&a, stream);
}

size_t zq_quantize_workspace_bytes(void) { return 256; }

int zq_quantize_fp8(const void* x, int x_dtype, int64_t n_vec, int d, int hadamard,
                    void* x_fp8, float* descale, void* workspace, void* stream) {
  if (!descale || !workspace) return ZQ_ERR_NULL;
  if (n_vec < 0 || d <= 0) return ZQ_ERR_SHAPE;
  if (n_vec > 0 && (!x || !x_fp8)) return ZQ_ERR_NULL;
  if (x_dtype != ZQ_X_F32 && x_dtype != ZQ_X_BF16) return ZQ_ERR_UNSUPPORTED;
  if (d % 8 != 0 || (hadamard && d % 128 != 0 && d != 192)) return ZQ_ERR_UNSUPPORTED;
  if (n_vec > (int64_t)1 << 40 || n_vec * (int64_t)d > ((int64_t)1 << 40)) return ZQ_ERR_SHAPE;
  if (!aligned16(x) || !aligned16(x_fp8) || !aligned16(workspace)) return ZQ_ERR_ALIGN;
  int sms = 0;
  int rc = check_device(&sms);
  if (rc != ZQ_OK) return rc;
  cudaError_t e = zq::launch_quantize(x, x_dtype == ZQ_X_BF16, n_vec * (int64_t)d,
                                      hadamard ? (d % 128 == 0 ? 1 : 2) : 0, x_fp8, descale, workspace,
                                      static_cast<cudaStream_t>(stream), sms);
  return e == cudaSuccess ? ZQ_OK : ZQ_ERR_CUDA;
}

size_t zq_quantize_multi_workspace_bytes(void) { return 256; }

int zq_quantize_fp8_multi(const zq_quant_tensor* t, int count, void* workspace, void* stream) {
  if (!t || !workspace) return ZQ_ERR_NULL;
  if (count < 1 || count > zq::kMaxQuantItems) return ZQ_ERR_SHAPE;
  zq::QuantItems Q = {};
  for (int i = 0; i < count; ++i) {
    const zq_quant_tensor& a = t[i];
    if (!a.descale) return ZQ_ERR_NULL;
    if (a.n_vec < 0 || a.d <= 0) return ZQ_ERR_SHAPE;
    if (a.n_vec > 0 && (!a.x || !a.x_fp8)) return ZQ_ERR_NULL;
    if (a.x_dtype != ZQ_X_F32 && a.x_dtype != ZQ_X_BF16) return ZQ_ERR_UNSUPPORTED;
    if (a.d % 8 != 0 || (a.hadamard && a.d % 128 != 0 && a.d != 192)) return ZQ_ERR_UNSUPPORTED;
    if (a.n_vec > (int64_t)1 << 40 || a.n_vec * (int64_t)a.d > ((int64_t)1 << 40)) return ZQ_ERR_SHAPE;
    if (!aligned16(a.x) || !aligned16(a.x_fp8)) return ZQ_ERR_ALIGN;
    Q.it[i].x = a.x;
    Q.it[i].out = static_cast<uint8_t*>(a.x_fp8);
    Q.it[i].descale = a.descale;
    Q.it[i].n = a.n_vec * (int64_t)a.d;
    Q.it[i].bf16 = a.x_dtype == ZQ_X_BF16 ? 1 : 0;
    Q.it[i].had = a.hadamard ? (a.d % 128 == 0 ? 1 : 2) : 0;
  }
  if (!aligned16(workspace)) return ZQ_ERR_ALIGN;
  int sms = 0;
  int rc = check_device(&sms);
  if (rc != ZQ_OK) return rc;
  cudaError_t e = zq::launch_quantize_multi(Q, count, workspace, static_cast<cudaStream_t>(stream), sms);
  return e == cudaSuccess ? ZQ_OK : ZQ_ERR_CUDA;
}

int zq_quantize_fp8_noalloc(const void* x, int x_dtype, int64_t n_vec, int d, int hadamard,
                            void* x_fp8, float* descale, void* stream) {
  if (!descale) return ZQ_ERR_NULL;
  if (n_vec < 0 || d <= 0) return ZQ_ERR_SHAPE;
  if (n_vec > 0 && (!x || !x_fp8)) return ZQ_ERR_NULL;
  if (x_dtype != ZQ_X_F32 && x_dtype != ZQ_X_BF16) return ZQ_ERR_UNSUPPORTED;
  if (d % 8 != 0 || (hadamard && d % 128 != 0 && d != 192)) return ZQ_ERR_UNSUPPORTED;
  if (n_vec > (int64_t)1 << 40 || n_vec * (int64_t)d > ((int64_t)1 << 40)) return ZQ_ERR_SHAPE;
  // the scratch this call needs must fit the fixed device array
  if (zq_quantize_workspace_bytes() > zq::noalloc_scratch_capacity()) return ZQ_ERR_SHAPE;
  if (!aligned16(x) || !aligned16(x_fp8)) return ZQ_ERR_ALIGN;
  int sms = 0;
  int rc = check_device(&sms);
  if (rc != ZQ_OK) return rc;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ZQ_ERR_CUDA;
  void* scratch = zq::noalloc_scratch_for_device(dev);
  if (!scratch) return ZQ_ERR_CUDA;
  cudaError_t e = zq::launch_quantize(x, x_dtype == ZQ_X_BF16, n_vec * (int64_t)d,
                                      hadamard ? (d % 128 == 0 ? 1 : 2) : 0, x_fp8, descale, scratch,
                                      static_cast<cudaStream_t>(stream), sms);
  return e == cudaSuccess ? ZQ_OK : ZQ_ERR_CUDA;
}

size_t zq_quantize_noalloc_scratch_bytes(void) { return zq::noalloc_scratch_capacity(); }

size_t zq_quantize_grouped_workspace_bytes(int B, int H, int heads_per_scale) {
  if (B <= 0 || H <= 0 || heads_per_scale <= 0 || H % heads_per_scale != 0) return 0;
  const int64_t slots = (int64_t)B * (H / heads_per_scale);
  if (slots > kMaxGroupedSlots) return 0;
  return (size_t)((slots * 4 + 15) / 16 * 16);
}

int zq_quantize_fp8_grouped(const void* x, int x_dtype, int B, int64_t S, int H, int d,
                            int heads_per_scale, int hadamard, void* x_fp8, float* descale,
                            void* workspace, void* stream) {
  if (!descale || !workspace) return ZQ_ERR_NULL;
  if (B <= 0 || H <= 0 || S < 0 || d <= 0 || heads_per_scale <= 0) return ZQ_ERR_SHAPE;
  if (H % heads_per_scale != 0) return ZQ_ERR_SHAPE;
  if ((int64_t)B * (H / heads_per_scale) > kMaxGroupedSlots) return ZQ_ERR_SHAPE;
  if (S > 0 && (!x || !x_fp8)) return ZQ_ERR_NULL;
  if (x_dtype != ZQ_X_F32 && x_dtype != ZQ_X_BF16) return ZQ_ERR_UNSUPPORTED;
  if (d % 8 != 0 || (hadamard && d % 128 != 0 && d != 192)) return ZQ_ERR_UNSUPPORTED;
  if (S > ((int64_t)1 << 40) || (int64_t)H * d > ((int64_t)1 << 24) ||
      (int64_t)B * S > ((int64_t)1 << 40) / ((int64_t)H * d))
    return ZQ_ERR_SHAPE;
  if (!aligned16(x) || !aligned16(x_fp8) || !aligned16(workspace)) return ZQ_ERR_ALIGN;
  int sms = 0;
  int rc = check_device(&sms);
  if (rc != ZQ_OK) return rc;
  cudaError_t e = zq::launch_quantize_grouped(
      x, x_dtype == ZQ_X_BF16, B, S, H, d, heads_per_scale,
      hadamard ? (d % 128 == 0 ? 1 : 2) : 0, x_fp8, descale, workspace,
      static_cast<cudaStream_t>(stream), sms);
  return e == cudaSuccess ? ZQ_OK : ZQ_ERR_CUDA;
}

int zq_debug_exp2(const float* x, float* y, int64_t n, int degree, void* stream) {
  if (n < 0) return ZQ_ERR_SHAPE;
  if (n > 0 && (!x || !y)) return ZQ_ERR_NULL;
  if (degree != 3 && degree != 4 && degree != 0 && degree != -1) return ZQ_ERR_UNSUPPORTED;
  int rc = check_device(nullptr);
  if (rc != ZQ_OK) return rc;
  cudaError_t e = zq::launch_exp2_check(x, y, n, degree, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? ZQ_OK : ZQ_ERR_CUDA;
}

}  // extern "C"
