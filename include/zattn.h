/*
 * zattn.h -- C ABI of the B200 (sm_100a) causal prefill attention library.
 *
 * Operations follow the ZYFA announcement as re-reported by three web pages:
 *   [P1] "Zyphra ZYFA : FlashAttention en FP8 pour l'AMD MI355X, jusqu'a
 *        1,76 fois plus rapide" (lefilia.fr), paragraphs 1-3.
 *   [P2] "Zyphra rilascia ZYFA, kernel di attenzione FP8 ottimizzati per le
 *        GPU AMD" (aicronaca.it), sections "Che cosa ha annunciato Zyphra"
 *        and "Perche l'FP8 non basta da solo".
 *   [P3] "Zyphra ZYFA ... FP8 FlashAttention for AMD MI355X up to 1.76x"
 *        (ai4bro.com), sections TL;DR and "How ZYFA works".
 *
 * Conventions shared by every entry point
 *   - Pointers named q, k, v, out, lse, x, x_fp8, descale, workspace and
 *     status are DEVICE pointers on the current CUDA device; the caller owns
 *     all of them.  The library allocates nothing and keeps no state between
 *     calls besides two lookup caches (the driver's tensor-map encoder, and
 *     per device the address of the fixed scratch array of
 *     zq_quantize_fp8_noalloc), both filled atomically; it is safe to call
 *     from several host threads.
 *   - `stream` is a cudaStream_t passed as void*; NULL is the legacy default
 *     stream.  Every call is asynchronous on that stream and never
 *     synchronises.
 *   - Return value: ZQ_OK (0) or a negative ZQ_ERR_* code.  On an argument
 *     error nothing is launched and no output is written.  ZQ_ERR_CUDA means
 *     a launch failed (cudaGetLastError is left set for the caller).
 */
#ifndef ZATTN_H_
#define ZATTN_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define ZQ_API __attribute__((visibility("default")))
#else
#define ZQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* ---- element types ---- */
#define ZQ_DTYPE_BF16 0      /* q, k, v bfloat16 */
#define ZQ_DTYPE_FP8_E4M3 1  /* q, k, v OCP e4m3fn bytes with fp32 descales */

#define ZQ_X_F32 0  /* quantiser input fp32 */
#define ZQ_X_BF16 1 /* quantiser input bfloat16 */

/* ---- FP8 softmax modes ---- */
#define ZQ_SOFTMAX_EXACT 0 /* P~ = e4m3_rne(exp2(y - e))                   */
#define ZQ_SOFTMAX_LEANP 1 /* P~ bits = clamp(rne(8 (y - e)) + 56, 0, 126) */

/* ---- FP8 descale layouts (zq_attn_args.descale_layout) ---- */
#define ZQ_DESCALE_PER_TENSOR 0  /* q/k/v_descale each point to one fp32        */
#define ZQ_DESCALE_PER_KV_HEAD 1 /* each points to B * Hkv fp32, [b * Hkv + g] */

/* ---- status codes ---- */
#define ZQ_OK 0
#define ZQ_ERR_NULL (-1)        /* a required pointer is NULL              */
#define ZQ_ERR_SHAPE (-2)       /* a size <= 0, Hq % Hkv != 0, overflow    */
#define ZQ_ERR_UNSUPPORTED (-3) /* head dims, dtype, mode or option        */
#define ZQ_ERR_ALIGN (-4)       /* a pointer is not 16-byte aligned        */
#define ZQ_ERR_ARCH (-5)        /* current device is not sm_100            */
#define ZQ_ERR_CUDA (-6)        /* a CUDA driver/runtime call failed       */
#define ZQ_ERR_TIMEOUT (-7)     /* a device-side wait ran out (status word) */

/*
 * zq_attn_fwd -- causal (or full) forward prefill attention,
 *   out = softmax(q k^T * softmax_scale + mask) v,  lse = logsumexp per row.
 * [P3 TL;DR: causal forward (prefill) attention in FP8 e4m3 and BF16, head
 *  dim 128 and the MLA 192/128 shape; P2 "Che cosa ha annunciato Zyphra":
 *  a drop-in for flash_attn_func.]
 *
 *   q    (B, Sq, Hq,  d_qk) contiguous, bf16 or e4m3 bytes
 *   k    (B, Sk, Hkv, d_qk) contiguous, same type
 *   v    (B, Sk, Hkv, d_v)  contiguous, same type
 *   out  (B, Sq, Hq,  d_v)  contiguous bfloat16 (both input types)
 *   lse  (B, Hq, Sq) fp32 natural log, or NULL to skip
 *   (d_qk, d_v) in {(128,128), (192,128)};  Hq % Hkv == 0, query head h
 *   reads kv head h / (Hq / Hkv) (GQA).
 *   softmax_scale <= 0 selects 1/sqrt(d_qk).
 *   causal != 0: key c is visible to query i iff c <= i + Sk - Sq
 *   (bottom-right alignment); a query row with no visible key gets out = 0,
 *   lse = -inf.
 *   q/k/v_descale: device pointers to one fp32 each (per-tensor dequant
 *   scale, FP8 only; NULL means 1.0); ignored for bf16.  Per-(batch, kv
 *   head) descales go through zq_attn_fwd_ex (descale_layout).
 *   FP8 uses Lean P with per-(row, 64-key block) power-of-2 scaling and
 *   headroom 8 (see zq_attn_fwd_ex for the other modes).
 * Errors: ZQ_ERR_NULL (q, k, v or out NULL), ZQ_ERR_SHAPE, ZQ_ERR_UNSUPPORTED,
 *   ZQ_ERR_ALIGN (q, k, v, out, lse not 16-byte aligned), ZQ_ERR_ARCH,
 *   ZQ_ERR_CUDA.
 */
ZQ_API int zq_attn_fwd(const void* q, const void* k, const void* v, void* out, float* lse, int B,
                int Sq, int Sk, int Hq, int Hkv, int d_qk, int d_v, float softmax_scale,
                int causal, int dtype, const float* q_descale, const float* k_descale,
                const float* v_descale, void* stream);

/* Extended arguments for zq_attn_fwd_ex.  Fields up to v_descale have the
 * meaning given for zq_attn_fwd. */
typedef struct zq_attn_args {
  const void* q;
  const void* k;
  const void* v;
  void* out;
  float* lse;
  int B, Sq, Sk, Hq, Hkv, d_qk, d_v;
  float softmax_scale;
  int causal;
  int dtype;
  const float* q_descale;
  const float* k_descale;
  const float* v_descale;
  /* FP8 only.  softmax_mode: ZQ_SOFTMAX_EXACT or ZQ_SOFTMAX_LEANP
   * [P1 paragraph 3, P2 "Perche l'FP8 non basta da solo": Lean P replaces the
   * exponential by a multiply-add whose result is read as e4m3 bits]. */
  int softmax_mode;
  /* FP8 only.  1: every 64-key block of a row gets its own power-of-2
   * exponent e = ceil(block max of y) - headroom_T, absorbed by the block-
   * scaled PV matrix instruction [P1 paragraph 3; P3 "How ZYFA works" item
   * 3].  0: one running exponent per row (ceil of the running max minus
   * headroom_T), shared by all blocks. */
  int block_scale;
  /* FP8 only, 0..8: where the block maximum lands, 2^(T-1) < p~max <= 2^T. */
  int headroom_T;
  /* Optional device int.  Must hold 0 before the call; a device-side wait
   * that runs out writes ZQ_ERR_TIMEOUT there and the kernel returns early
   * (outputs are then undefined).  NULL: not reported. */
  int* status;
  /* FP8 only.  ZQ_DESCALE_PER_TENSOR (0): q/k/v_descale each point to one
   * fp32.  ZQ_DESCALE_PER_KV_HEAD (1): each points to B * Hkv fp32, row-major
   * (batch, kv head); query head h of batch b is dequantised with
   * q_descale[b * Hkv + h / (Hq / Hkv)], and its keys and values with the
   * k_descale / v_descale entry of the same index.  This is the (batch,
   * kv head) descale shape of flash_attn_func's FP8 interface, which the
   * kernel is a drop-in for [P2 "Che cosa ha annunciato Zyphra"];
   * zq_quantize_fp8_grouped produces such scales.  NULL pointers still
   * mean 1.0. */
  int descale_layout;
} zq_attn_args;

/* zq_attn_fwd_ex -- zq_attn_fwd with the options above.  Same errors, plus
 * ZQ_ERR_UNSUPPORTED for softmax_mode / block_scale / headroom_T out of
 * range (they are ignored, not checked, for bf16). */
ZQ_API int zq_attn_fwd_ex(const zq_attn_args* args, void* stream);

/* Launch shape of one attention call, from zq_attn_plan_launch. */
typedef struct zq_attn_plan {
  int64_t n_units;   /* work units: ceil(Sq / rows_per_unit) x B x Hq          */
  int64_t grid;      /* CTAs launched                                          */
  int persistent;    /* 1: each CTA walks several units (Sq <= 64 x 128 rows)  */
  int head_group;    /* flat heads whose tiles are interleaved in unit order  */
  int smem_bytes;    /* dynamic shared memory per CTA                          */
  int threads;       /* threads per CTA                                        */
  int rows_per_unit; /* query rows per unit: 128, or 256 (BF16 at d_qk = d_v =
                        128: a pair of 128-row tiles, one per softmax team)    */
  int keys_per_tile; /* keys per key tile: 128, or 64 with 256-row units       */
} zq_attn_plan;

/*
 * zq_attn_plan_launch -- the schedule zq_attn_fwd_ex would launch for `args`,
 * computed on the host (host code only; nothing is launched or read from
 * the device).
 * [P3 TL;DR: causal prefill -- a query tile visits only key tiles holding a
 *  key visible to one of its rows; GQA maps query head h to kv head
 *  h / (Hq / Hkv).]
 *
 *   args      validated exactly as by zq_attn_fwd_ex (same errors); the
 *             device pointers in it are not dereferenced.
 *   num_sms   SMs to plan for; <= 0 asks the current device (which must
 *             then be sm_100, else ZQ_ERR_ARCH / ZQ_ERR_CUDA).
 *   plan      receives the launch shape.
 *   unit_tile, unit_bh, unit_nkv, unit_cta, unit_round: optional HOST
 *             arrays of plan->n_units int32 each (NULL to skip; call once
 *             with all NULL to learn n_units).  Entry u describes work unit
 *             u: its index t along the query axis (rows
 *             rows_per_unit * t ..  + rows_per_unit - 1), its flat head
 *             b * Hq + h, the number of key tiles of keys_per_tile keys it
 *             visits (tiles 0..n_kv-1; with 256-row units the later 128-row
 *             tile's count, the earlier one stopping at its own diagonal),
 *             the CTA that runs it and its position in that CTA's
 *             sequence.  Units are numbered in groups of head_group
 *             heads, longest rows first inside a group; a persistent CTA c
 *             of G runs, in round k, unit k*G + c (k even) or
 *             k*G + G-1-c (k odd).
 * Errors: ZQ_ERR_NULL (plan NULL, or as zq_attn_fwd_ex), ZQ_ERR_SHAPE,
 *   ZQ_ERR_UNSUPPORTED, ZQ_ERR_ALIGN, ZQ_ERR_ARCH, ZQ_ERR_CUDA.
 */
ZQ_API int zq_attn_plan_launch(const zq_attn_args* args, int num_sms, zq_attn_plan* plan,
                               int32_t* unit_tile, int32_t* unit_bh, int32_t* unit_nkv,
                               int32_t* unit_cta, int32_t* unit_round);

/* zq_attn_fwd_debug -- zq_attn_fwd_ex that also dumps, for the query tile
 * dbg_qtile (rows 128*dbg_qtile..) of flat head dbg_bh = batch*Hq + head,
 * the first 128x128 score tile before masking and the
 * P words written for it, to the device buffer `dbg` (caller-owned,
 * ZQ_DEBUG_BYTES bytes): float S[128][128] (raw q.k dot products, no
 * scale), uint32 P[128][64] (bf16: 64 words of 2 x bf16; FP8: the first 32
 * words hold 4 x e4m3 each, key order little-endian), uint32 SF[2][128]
 * (FP8: the UE8M0 scale of 64-key block 0 / 1 of each row, repeated in all
 * four bytes), then uint64 TRACE[512][16]: SM clock (clock64) at up to sixteen points of
 * the pipeline for key tile j (see attn_fwd.cu); with 256-row units
 * (zq_attn_plan.rows_per_unit, BF16 at d = 128) TRACE[512][2][8] for 64-key
 * tile j, the traced tile's team t = dbg_qtile & 1 in [j][t] (see
 * attn_pp.cu).  flags: 0, or 1 to make
 * the MMA issuers withhold all work so that every other role's bounded wait
 * runs out: the kernel then writes ZQ_ERR_TIMEOUT to args->status and
 * returns (about two seconds later) with the outputs undefined; nothing
 * faults or hangs.  For tests and tuning. */
#define ZQ_DEBUG_BYTES (128 * 128 * 4 + 128 * 64 * 4 + 256 * 4 + 512 * 16 * 8)
ZQ_API int zq_attn_fwd_debug(const zq_attn_args* args, void* dbg, int dbg_bh, int dbg_qtile,
                             int flags, void* stream);

/*
 * zq_quantize_fp8 -- per-tensor FP8 e4m3 quantiser with an optional fused
 * 128-point Walsh-Hadamard rotation [P2 "Perche l'FP8 non basta da solo":
 * a Hadamard rotation of Q and K roughly halves the input quantisation error].
 *
 *   x        n_vec vectors of d channels, fp32 (x_dtype ZQ_X_F32) or bf16
 *   hadamard != 0: every 128-channel slice is replaced by H_128 x (Sylvester
 *            order, entries +-1, fp32 butterflies at strides 1,2,...,64);
 *            requires d % 128 == 0, or d == 192 (the MLA query/key width):
 *            then channels 128..191 are replaced by sqrt(2) H_64 x (fp32
 *            butterflies at strides 1..32, then each value times
 *            fl32(sqrt 2)), which scales scores by 128 like H_128.
 *   amax     = max |x| (after rotation);  inv = fl32(448 / amax)
 *   x_fp8    (n_vec, d) e4m3 bytes = e4m3_rne_satfinite(fl32(x * inv))
 *   descale  one fp32 = fl32(amax / 448), times fl32(2^-3.5) when rotated,
 *            so that (H q)(H k)^T descales to q k^T.  amax == 0 gives all-
 *            zero codes and descale 0.
 *   workspace  device scratch of zq_quantize_workspace_bytes() bytes, 16-byte
 *            aligned; its contents on entry do not matter and it must not be
 *            used by another call that runs at the same time.
 * n_vec == 0 writes only the descale (0); x and x_fp8 may then be NULL.
 * Errors: ZQ_ERR_NULL, ZQ_ERR_SHAPE (n_vec < 0, d <= 0), ZQ_ERR_UNSUPPORTED
 *   (x_dtype, hadamard with d % 128 != 0 and d != 192, d % 8 != 0), ZQ_ERR_ALIGN (x,
 *   x_fp8, workspace not 16-byte aligned), ZQ_ERR_ARCH, ZQ_ERR_CUDA.
 */
ZQ_API int zq_quantize_fp8(const void* x, int x_dtype, int64_t n_vec, int d, int hadamard,
                    void* x_fp8, float* descale, void* workspace, void* stream);

/* Bytes of device scratch zq_quantize_fp8 needs (a small constant). */
ZQ_API size_t zq_quantize_workspace_bytes(void);

/*
 * zq_quantize_fp8_multi -- zq_quantize_fp8 applied to `count` tensors at
 * once (1 <= count <= 4; the query, key and value inputs of one attention
 * call), each with its own scale.  [P2 "Perche l'FP8 non basta da solo": the
 * inputs are quantised per tensor, with the rotation on Q and K only.]
 *
 *   t[i]     one tensor: the arguments of zq_quantize_fp8 (x, x_dtype,
 *            n_vec, d, hadamard, x_fp8, descale), validated the same way;
 *            every tensor's bytes and descale equal what zq_quantize_fp8
 *            writes for it alone.
 *   workspace  device scratch of zq_quantize_multi_workspace_bytes() bytes,
 *            16-byte aligned; its contents on entry do not matter and it must
 *            not be used by another call that runs at the same time.
 * The call makes three stream operations in all (a clear of `count` words and
 * two kernels) instead of three per tensor.  Outputs must not overlap inputs
 * or each other.
 * Errors: those of zq_quantize_fp8 for any tensor; ZQ_ERR_NULL (t or
 *   workspace NULL), ZQ_ERR_SHAPE (count outside 1..4).
 */
typedef struct zq_quant_tensor {
  const void* x;
  int x_dtype;
  int64_t n_vec;
  int d;
  int hadamard;
  void* x_fp8;
  float* descale;
} zq_quant_tensor;

ZQ_API int zq_quantize_fp8_multi(const zq_quant_tensor* t, int count, void* workspace, void* stream);

/* Bytes of device scratch zq_quantize_fp8_multi needs (a small constant). */
ZQ_API size_t zq_quantize_multi_workspace_bytes(void);

/*
 * zq_quantize_fp8_noalloc -- zq_quantize_fp8 without a workspace argument.
 * (The pages describe no counterpart; this is a library convenience.)
 *
 * For callers that cannot provide device scratch memory: hosts whose device
 * memory belongs to another allocator that offers no scratch API, and
 * latency-critical loops that must not call cudaMalloc because it can
 * synchronise the device.  The scratch lives instead in one fixed device
 * array inside this library, zq_quantize_noalloc_scratch_bytes() bytes
 * (256), which every GPU that loads the library holds until the process
 * exits.  The quantiser needs 256 bytes whatever the input size, so every
 * input the regular entry point accepts fits; a request for more scratch
 * than the array holds is rejected with ZQ_ERR_SHAPE.
 *
 * Arguments, outputs and the other errors are those of zq_quantize_fp8.
 * The call allocates nothing (no cudaMalloc / cudaFree or allocating library
 * routine).  The first call on each device looks up the array's device
 * address with that device current and caches it; make that first call
 * before any stream capture.  All calls share the one array and it keeps the
 * last call's contents (the amax word is cleared at the start of each call),
 * so calls whose work can overlap on the GPU -- on different streams without
 * ordering between them -- race and must not be issued that way.
 * The cached address belongs to the device's primary context as it was at
 * the first call: a device reset (cudaDeviceReset) or any other teardown of
 * that context invalidates it, and calling this entry point on the device
 * afterwards in the same process is not supported.
 */
ZQ_API int zq_quantize_fp8_noalloc(const void* x, int x_dtype, int64_t n_vec, int d, int hadamard,
                                   void* x_fp8, float* descale, void* stream);

/* Capacity in bytes of the fixed scratch array of zq_quantize_fp8_noalloc. */
ZQ_API size_t zq_quantize_noalloc_scratch_bytes(void);

/*
 * zq_quantize_fp8_grouped -- the quantiser of zq_quantize_fp8 with one scale
 * per (batch, group of heads) instead of one per tensor.
 *
 *   x        (B, S, H, d) contiguous, fp32 or bf16 (x_dtype)
 *   heads_per_scale  g: heads [gi*g, gi*g + g) of batch b form slot
 *            b * (H / g) + gi.  Queries take g = Hq / Hkv and keys and
 *            values g = 1, which gives the ZQ_DESCALE_PER_KV_HEAD layout of
 *            zq_attn_args.
 *   Each slot, x[b, :, heads of the slot, :], is quantised exactly as
 *   zq_quantize_fp8 quantises a whole tensor (same rotation, same rounding,
 *   its own amax): codes bit-identical to zq_quantize_fp8 run on that slot
 *   alone.
 *   x_fp8    (B, S, H, d) e4m3 bytes
 *   descale  B * (H / g) fp32, row-major (batch, slot)
 *   workspace  device scratch of zq_quantize_grouped_workspace_bytes(B, H, g)
 *            bytes, 16-byte aligned, not shared with a concurrent call.
 * S == 0 writes only the descales (0); x and x_fp8 may then be NULL.
 * Errors: ZQ_ERR_NULL, ZQ_ERR_SHAPE (B, H, d, g <= 0, S < 0, H % g != 0,
 *   more than 65535 slots, size overflow), ZQ_ERR_UNSUPPORTED (as for
 *   zq_quantize_fp8), ZQ_ERR_ALIGN (x, x_fp8, workspace), ZQ_ERR_ARCH,
 *   ZQ_ERR_CUDA.
 */
ZQ_API int zq_quantize_fp8_grouped(const void* x, int x_dtype, int B, int64_t S, int H, int d,
                                   int heads_per_scale, int hadamard, void* x_fp8, float* descale,
                                   void* workspace, void* stream);

/* Bytes of device scratch zq_quantize_fp8_grouped needs for these sizes
 * (4 per slot, rounded up to 16); 0 for arguments it would reject. */
ZQ_API size_t zq_quantize_grouped_workspace_bytes(int B, int H, int heads_per_scale);

/* zq_debug_exp2 -- y[i] = 2^x[i] by the kernels' software exp2 (degree 3 or
 * 4 minimax polynomial after range reduction), by CUDA's exp2f (degree 0) or
 * by the hardware approximation ex2.approx (degree -1).  x, y: device fp32
 * arrays of n elements.  For the test that bounds the polynomial's error
 * against exp2f.  Errors: ZQ_ERR_SHAPE, ZQ_ERR_NULL, ZQ_ERR_UNSUPPORTED,
 * ZQ_ERR_ARCH, ZQ_ERR_CUDA. */
ZQ_API int zq_debug_exp2(const float* x, float* y, int64_t n, int degree, void* stream);

/* Static text for a status code (never NULL). */
ZQ_API const char* zq_status_string(int status);

/* Library version as major*10000 + minor*100 + patch. */
ZQ_API int zq_version(void);

#ifdef __cplusplus
}
#endif
#endif /* ZATTN_H_ */
