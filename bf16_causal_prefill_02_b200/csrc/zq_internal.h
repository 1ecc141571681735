// zq_internal.h -- launch structures shared by the C-ABI layer and the
// kernels (internal; not part of the public interface).
#pragma once
#include <cuda_runtime.h>

#include <cstdint>

namespace zq {

struct AttnParams {
  void* out;  // (B, Sq, Hq, d_v) bfloat16
  float* lse;  // (B, Hq, Sq) or nullptr
  const float* q_descale;
  const float* k_descale;
  const float* v_descale;
  // 0: each descale pointer holds one fp32; 1: each holds B * Hkv fp32,
  // entry b * Hkv + kv_head (query head h uses kv head h / (Hq / Hkv))
  int descale_per_kv;
  int* status;
  int B, Sq, Sk, Hq, Hkv;
  int n_qtiles;
  // Block order: blocks come in groups of head_group consecutive flat heads
  // (head_group divides B * Hq); inside a group, query tiles run longest
  // causal rows first, interleaved across the group's heads.  head_group =
  // B * Hq is plain longest-rows-first over all heads; a small group keeps
  // the blocks that run together on few heads, so their K/V tiles are
  // shared in L2.
  int head_group;
  int causal;
  int headroom_T;
  float softmax_scale;
  uint64_t timeout_ns;
  // Debug dump (nullptr in normal use): the CTA of flat (batch*Hq + head)
  // dbg_bh and query tile dbg_t writes its first score tile, P words and
  // scale words here: float S[128][128]; uint32 P[128][64]; uint32 SF[2][128].
  void* dbg;
  int dbg_bh, dbg_t;
  // Test hook: bit 0 makes the MMA issuer withhold all work, so every other
  // role's wait runs into its time limit and the kernel reports
  // ZQ_ERR_TIMEOUT through the status word (exercises the failure path
  // without faulting or hanging the GPU).
  int dbg_flags;
};

struct AttnLaunch {
  const void* q;
  const void* k;
  const void* v;
  AttnParams p;
  int dqk, dv, dtype, mode, block_scale;
};

cudaError_t launch_attention(const AttnLaunch& a, cudaStream_t st);
// the paired kernel (two 128-row query tiles per CTA, 64-key tiles, one
// CTA per unit): BF16 at d_qk = d_v = 128 with more than 64 query tiles;
// launch_attention dispatches to it
bool use_pair_kernel(int dtype, int dqk, int n_qtiles);
cudaError_t launch_attention_pp(const AttnLaunch& a, cudaStream_t st);
int attn_pp_smem_bytes();
int attn_pp_threads();
// dynamic shared memory and threads of one attention CTA (host side)
int attn_smem_bytes(int dtype, int dqk);
int attn_threads();
// hadamard: 0 none, 1 H128 on every 128-slice (d % 128 == 0), 2 the d = 192
// rotation (H128 on channels 0..127, sqrt2 * H64 on 128..191)
cudaError_t launch_quantize(const void* x, int x_bf16, int64_t n, int hadamard, void* out,
                            float* descale, void* workspace, cudaStream_t st, int num_sms);
// x (B, S, H, d); heads [gi*g, gi*g + g) of batch b share one scale, slot
// b*(H/g) + gi; hadamard as for launch_quantize.
cudaError_t launch_quantize_grouped(const void* x, int x_bf16, int B, int64_t S, int H, int d, int g,
                                    int hadamard, void* out, float* descale, void* workspace,
                                    cudaStream_t st, int num_sms);
// One tensor of a multi-tensor quantiser call: n elements (n % 4 == 0; for
// had == 2, n % 192 == 0), bf16 input or fp32, had 0 none / 1 H128 / 2 the
// d = 192 rotation.  `blocks` is filled in by the launcher.
struct QuantItem {
  const void* x;
  uint8_t* out;
  float* descale;
  int64_t n;
  int bf16, had, blocks;
};
constexpr int kMaxQuantItems = 4;
struct QuantItems {
  QuantItem it[kMaxQuantItems];
};
cudaError_t launch_quantize_multi(QuantItems Q, int count, void* workspace, cudaStream_t st, int num_sms);
void* noalloc_scratch_for_device(int dev);
cudaError_t launch_exp2_check(const float* x, float* y, int64_t n, int degree, cudaStream_t st);
size_t noalloc_scratch_capacity();

}  // namespace zq
