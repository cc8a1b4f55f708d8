/*
 * frt.h -- fused non-GEMM layer ops for B200 (sm_100a), C ABI of libfrt.so.
 *
 * Three fused ops cover the memory- and launch-bound chain that sits between
 * the GEMMs of a small-batch transformer layer ("FlashRT kernel fusion",
 * §二 per-layer table: steps 1/7, 3 and 8-10):
 *
 *   frt_residual_rmsnorm_fp8   residual add + RMSNorm + FP8 e4m3 quantisation
 *   frt_qkv_norm_rope_kvcache  packed-QKV split + per-head q/k RMSNorm +
 *                              rotate-half RoPE + Q staging + KV-cache write
 *   frt_gate_act_fp8           gated activation on interleaved gate/up + FP8
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Pointers marked "device" are caller-owned device memory; the library
 *    allocates nothing and keeps no pointer after the call returns.
 *  - Every call is asynchronous on `stream` (0 = legacy default stream), never
 *    synchronises, holds no state between calls and may be captured into a
 *    CUDA graph.
 *  - Host-detectable errors return a status before anything is launched:
 *      FRT_ERR_INVALID_ARG  negative sizes, a size that breaks the layout rule
 *                           stated per op, a required pointer that is NULL,
 *                           a pointer below its stated alignment, a missing
 *                           scale pointer for the chosen quant mode, an unknown
 *                           enum value;
 *      FRT_ERR_UNSUPPORTED  a valid shape this build does not cover (stated per
 *                           op);
 *      FRT_ERR_CUDA         the launch itself failed (cudaGetLastError after
 *                           the launch).
 *  - M == 0 is an empty batch: once the sizes and enum values pass their
 *    checks the call returns FRT_OK and launches nothing; pointers are not
 *    inspected (an empty tensor may have a NULL data pointer).
 *  - Device-side data errors never trap: see the status word of op (b).
 *  - 16-bit tensors are fp16 or bf16 as selected by `dt`; all layouts are
 *    row-major and contiguous.  e4m3 is OCP FP8 E4M3 ("fn": max 448, no inf).
 *  - FP8 conversion rounds to nearest-even and saturates to +-448; NaN input
 *    gives the NaN code.
 *  - Aliasing: only residual_out == residual_in (op a) is allowed; any other
 *    overlap between outputs, or between an output and an input, is undefined.
 */
#ifndef FRT_H_
#define FRT_H_

#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FRT_OK = 0,
  FRT_ERR_INVALID_ARG = 1,
  FRT_ERR_UNSUPPORTED = 2,
  FRT_ERR_CUDA = 3
} frt_status;

typedef enum { FRT_F16 = 0, FRT_BF16 = 1 } frt_dtype;

/* FP8 scaling.  A scale s is a dequantisation scale: code = e4m3(y / s), so
 * y ~ code * s.
 *  STATIC   one fp32 scale for the whole tensor, read from device memory
 *           ("FlashRT kernel fusion", §六: `_static` = constant activation
 *           scale).
 *  BLOCK128 per row and per 128-column block b = [128b, min(128b+128, N)):
 *           s = amax/448 over the block's valid columns (s = 1 for an all-zero
 *           block), written as fp32 to block_scales[row * ceil(N/128) + b]
 *           ("sm89 prefill FFN megakernel", Phase 2: per-token block-128 FP8
 *           and its out_scale).  Every scale of every row is written. */
typedef enum { FRT_QUANT_STATIC = 0, FRT_QUANT_BLOCK128 = 1 } frt_quant;

/* Gate activations, applied to the even element g of each (g, u) pair:
 *  GELU_TANH  0.5 g (1 + tanh(sqrt(2/pi) (g + 0.044715 g^3)))  (GeGLU)
 *  SILU       g / (1 + exp(-g))                                (SwiGLU)
 *  RELU2      max(g, 0)^2; any sqrt(2) factor is already in the gate weights
 *             ("Falcon-Perception inference optimisation", third technique). */
typedef enum { FRT_ACT_GELU_TANH = 0, FRT_ACT_SILU = 1, FRT_ACT_RELU2 = 2 } frt_act;

/* Scale-factor layout of the NVFP4 producers (NEXT-3):
 *  ROW_MAJOR       sf[M, N/16] row-major bytes
 *  SWIZZLED_128X4  the layout block-scaled tensor-core GEMMs read: 512-byte
 *                  atoms of 128 rows x 4 scale columns, laid out row-major over
 *                  (row / 128, column / 4) with ceil(N/64) atoms per atom row;
 *                  inside an atom, row 32 i + k and column l sit at byte
 *                  16 k + 4 i + l.  The array holds ceil(M/128) * 128 *
 *                  ceil(N/64) * 4 bytes; padding bytes are not written. */
typedef enum { FRT_SF_ROW_MAJOR = 0, FRT_SF_SWIZZLED_128X4 = 1 } frt_sf_layout;

/* Q staging layout of the QKV op with the Q epilogue (NEXT-2):
 *  TOKEN_MAJOR  q_out[M, Hq, hd]  (op (b)'s layout)
 *  HEAD_MAJOR   q_out[Hq, M, hd]  (one contiguous [M, hd] slab per head) */
typedef enum { FRT_Q_TOKEN_MAJOR = 0, FRT_Q_HEAD_MAJOR = 1 } frt_q_layout;

/* KV-cache element format of the QKV op with the Q epilogue (NEXT-2):
 *  16BIT  the op's 16-bit type (op (b))
 *  E4M3   FP8 e4m3 codes, one static dequantisation scale per tensor:
 *         code = e4m3(k / k_scale), e4m3(v / v_scale) */
typedef enum { FRT_KV_16BIT = 0, FRT_KV_E4M3 = 1 } frt_kv_format;

/*
 * (a) Residual add + RMSNorm + FP8 quantisation.
 * "FlashRT kernel fusion", §二 steps 1 and 7 (residual_add_rms_norm_fp8_noweight)
 * and §2.1 (the three element-wise steps share one pass over the row); §三 for
 * the `_noweight` form whose (1 + w) is folded into the next GEMM's weights.
 *
 * For each row i (M rows of D columns):
 *   h[i,j]   = x[i,j] + residual_in[i,j], the exact sum rounded once to the
 *              16-bit type (RNE); written to residual_out (the new residual
 *              stream).
 *   rstd_i   = 1 / sqrt(mean_j(h[i,j]^2) + eps), computed from the rounded h
 *              with fp64 accumulation (the squares are exact) in a fixed
 *              order.
 *   y[i,j]   = h[i,j] * rstd_i * weight[j]   (weight == NULL: no weight).
 *   out_fp8  = e4m3 of y / s (quant mode as above; block scales over D).
 *              The value converted is y / s rounded to fp32: with a static
 *              scale one rounding of h * w * (rstd / s), with block-128
 *              scales the correctly rounded quotient of the fp32 y.
 *
 *   x, residual_in, residual_out  device, [M, D] 16-bit, 16-byte aligned;
 *                                 residual_out may equal residual_in.
 *   weight        device [D] 16-bit, 16-byte aligned, or NULL.
 *   out_fp8       device [M, D] uint8, 8-byte aligned.
 *   static_scale  STATIC: device fp32[1], 4-byte aligned; else ignored.
 *   block_scales  BLOCK128: device fp32 [M, ceil(D/128)]; else ignored.
 *   Layout rule: D > 0 and D % 8 == 0.  Unsupported: D > 32768.
 */
frt_status frt_residual_rmsnorm_fp8(const void* x, const void* residual_in, void* residual_out,
                                    const void* weight, uint8_t* out_fp8, const float* static_scale,
                                    float* block_scales, int M, int D, float eps, frt_dtype dt,
                                    frt_quant qm, cudaStream_t stream);

/*
 * (b) Packed QKV split + per-head q/k RMSNorm + rotate-half RoPE + Q staging
 *     + KV-cache write.
 * "FlashRT kernel fusion", §2.2 first bullet (q_norm -> RoPE -> Q staging and
 * k_norm -> RoPE -> KV cache in one kernel; V passes straight through) and
 * second bullet (rotate_half RoPE with each rotation pair kept in one lane);
 * §二 step 3 (QKV split + RoPE + KV-cache write, no q/k norm); §四 (RoPE table
 * precomputed).
 *
 * Row i of qkv is [Q heads (Hq*hd) | K heads (Hkv*hd) | V heads (Hkv*hd)],
 * each head contiguous.  With p = positions[i] and half = hd/2:
 *   v      = one Q or K head, in fp32;
 *   norm   v = v * (1/sqrt(mean(v^2) + eps)) * w   with w = q_norm_w for Q
 *            heads, k_norm_w for K heads; skipped for a side whose weight is
 *            NULL (fp32; 1/sqrt by the hardware reciprocal square root,
 *            relative error about 2^-22);
 *   rope   for j < half, c = cos_tab[p, j], s = sin_tab[p, j]:
 *            o[j] = v[j] c - v[j+half] s,  o[j+half] = v[j+half] c + v[j] s;
 *   q_out[i, h, :]          = o (Q head h), rounded once to 16 bits;
 *   k_cache[p, g, :]        = o (K head g), rounded once to 16 bits;
 *   v_cache[p, g, :]        = V head g, bit copy.
 * The RoPE position is also the cache slot.  Duplicate positions within one
 * call leave the slot with one of the rows (which one is unspecified).
 *
 *   qkv                 device [M, (Hq+2Hkv)*hd] 16-bit.
 *   q_norm_w, k_norm_w  device [hd] 16-bit each, or NULL.
 *   cos_tab, sin_tab    device [max_pos, hd/2] fp32, 16-byte aligned.
 *   positions           device int32 [M].
 *   q_out               device [M, Hq, hd] 16-bit.
 *   k_cache, v_cache    device [capacity, Hkv, hd] 16-bit; rows other than the
 *                       M written slots are left untouched.
 *   status              device int32[1] or NULL.  Bits are set with an atomic
 *                       OR and never cleared by the call:
 *                       bit 0  a row's position is < 0, >= max_pos or
 *                              >= capacity; that row is skipped entirely (no
 *                              Q, K or V write);
 *                       bit 1  a kernel gave up waiting for its own bulk copy
 *                              (a bounded wait ran out: only a failing device,
 *                              or a bound lowered by frt_set_wait_polls, can
 *                              cause it); that token's outputs are not
 *                              written.
 *   16-bit pointers must be 16-byte aligned when hd % 16 == 0, 8-byte aligned
 *   when hd % 8 == 0, and 2-byte aligned otherwise (a head dim that no vector
 *   width divides, e.g. 66 or 100, runs an element-wise kernel); cos_tab and
 *   sin_tab 16-byte aligned when hd % 8 == 0, else 4-byte.
 *   Layout rule: Hq, Hkv > 0, Hq % Hkv == 0, hd > 0 and even, max_pos > 0,
 *   capacity > 0.  Unsupported: hd > 256.
 */
frt_status frt_qkv_norm_rope_kvcache(const void* qkv, const void* q_norm_w, const void* k_norm_w,
                                     const float* cos_tab, const float* sin_tab, const int32_t* positions,
                                     void* q_out, void* k_cache, void* v_cache, int32_t* status, int M,
                                     int Hq, int Hkv, int hd, int max_pos, int capacity, float eps,
                                     frt_dtype dt, cudaStream_t stream);

/*
 * (c) Gated activation on an interleaved gate/up buffer + FP8 quantisation.
 * "Falcon-Perception inference optimisation", third technique (the gate and
 * up weights are stored interleaved so one GEMM yields [g0,u0,g1,u1,...]; one
 * kernel reads each adjacent pair, computes relu(g)^2 * u and writes once);
 * "FlashRT kernel fusion", §二 steps 8-10 (GELU * up + quant, 3 -> 1);
 * "sm89 prefill FFN megakernel", Phase 2 (silu * mul + per-token block-128 FP8).
 *
 *   a[i,j]   = act(g) * u with g = gate_up[i, 2j], u = gate_up[i, 2j+1],
 *              in fp32 (GELU-tanh and SiLU through exp(x) = 2^(x log2 e) and
 *              1 / (1 + e) on the special-function unit's approximations,
 *              relative error about 2^-21).
 *   out_fp8  = e4m3 of a / s (quant mode as above; block scales over I).
 *
 *   gate_up       device [M, 2I] 16-bit, 16-byte aligned.
 *   out_fp8       device [M, I] uint8, 4-byte aligned.
 *   static_scale  STATIC: device fp32[1]; else ignored.
 *   block_scales  BLOCK128: device fp32 [M, ceil(I/128)]; else ignored.
 *   Layout rule: I > 0 and I % 4 == 0.
 */
frt_status frt_gate_act_fp8(const void* gate_up, uint8_t* out_fp8, const float* static_scale,
                            float* block_scales, int M, int I, frt_act act, frt_dtype dt, frt_quant qm,
                            cudaStream_t stream);

/*
 * NEXT-4: the layer chain as one persistent kernel (small batches).
 * "FlashFormer: Whole-Model Kernels for Efficient Low-Batch Inference" (the
 * whole sequence in one kernel); the chain is the graphed one: for each of
 * `steps` steps and each layer l, in order,
 *   frt_residual_rmsnorm_fp8(x_attn[l], residual, residual, w_attn[l], q8_attn[l], scales[0] / bs_attn[l])
 *   frt_qkv_norm_rope_kvcache(qkv[l], q_norm_w[l], k_norm_w[l], cos, sin, positions, q_out[l], k_cache[l], v_cache[l])
 *   frt_residual_rmsnorm_fp8(x_ffn[l], residual, residual, w_ffn[l], q8_ffn[l], scales[1] / bs_ffn[l])
 *   frt_gate_act_fp8(gate_up[l], act8[l], scales[2] / bs_act[l])
 * with the same results as those launches (the residual stream carries from
 * op to op).  Every op of the chain reads only its own row of each buffer, so
 * one CTA per row runs the row's whole chain in one launch.
 *
 *   layers      device array [n_layers] of frt_chain_layer (pointers as in the
 *               per-op calls; weights may be NULL; bs_* used with BLOCK128).
 *   residual    device [M, D] 16-bit, updated in place.
 *   scales      device fp32[3] (attention norm, FFN norm, activation), read
 *               with STATIC.
 *   status      device int32[1] or NULL; bits set with an atomic OR, never
 *               cleared: bit 0 as op (b) (a row's position out of range:
 *               that row's QKV outputs are skipped); bit 2 a layer record
 *               holds a pointer below its field's alignment (16 bytes for the
 *               eight inputs, k_cache, v_cache and q_out, 8 for q8_attn and
 *               q8_ffn, 4 for act8 and bs_*), checked in the kernel before
 *               anything is read or written: the launch then writes nothing.
 *   Supported: D % 8 == 0 and D <= 8192, hd % 16 == 0 and 64 <= hd <= 256,
 *   I % 128 == 0 (else FRT_ERR_UNSUPPORTED).  residual, cos_tab and sin_tab
 *   16-byte aligned, positions and scales 4-byte (checked on the host).
 *   Each row is run by a thread-block cluster of up to 8 CTAs, sized so that
 *   the clusters of all M rows fill the GPU: one runs the row's residual chain
 *   (the norms), the others split the heads and activation blocks and run
 *   alongside it.
 */
typedef struct frt_chain_layer {
  const void* x_attn;   /* [M, D] */
  const void* x_ffn;    /* [M, D] */
  const void* w_attn;   /* [D] or NULL */
  const void* w_ffn;    /* [D] or NULL */
  const void* qkv;      /* [M, (Hq+2Hkv) hd] */
  const void* q_norm_w; /* [hd] or NULL */
  const void* k_norm_w; /* [hd] or NULL */
  const void* gate_up;  /* [M, 2I] interleaved */
  void* k_cache;        /* [capacity, Hkv, hd] */
  void* v_cache;        /* [capacity, Hkv, hd] */
  void* q_out;          /* [M, Hq, hd] */
  uint8_t* q8_attn;     /* [M, D] */
  uint8_t* q8_ffn;      /* [M, D] */
  uint8_t* act8;        /* [M, I] */
  float* bs_attn;       /* [M, ceil(D/128)] or NULL */
  float* bs_ffn;        /* [M, ceil(D/128)] or NULL */
  float* bs_act;        /* [M, I/128] or NULL */
} frt_chain_layer;

frt_status frt_chain_persistent(const frt_chain_layer* layers, int n_layers, int steps, void* residual,
                                const float* cos_tab, const float* sin_tab, const int32_t* positions,
                                const float* scales, int32_t* status, int M, int D, int Hq, int Hkv, int hd, int I,
                                int max_pos, int capacity, float eps, frt_dtype dt, frt_quant qm, frt_act act,
                                cudaStream_t stream);

/*
 * NEXT-4: LayerNorm variants.
 *
 * frt_residual_layernorm_fp8 / _nvfp4: the ViT "add_layer_norm" producer (the
 * FlashRT port's census: add_layer_norm_to_nvfp4).  Op (a) / its NVFP4 form
 * with LayerNorm in place of RMSNorm:
 *   h = x + residual (rounded once, written back);
 *   y = (h - mean) / sqrt(var + eps) * weight + bias, mean and (biased) var
 *       over the row (one fp64 pass: var = E[h^2] - mean^2), y in fp32 with a
 *       few roundings (static FP8: 1 / s folded into the norm factor and the
 *       bias);
 *   then FP8 (static / block-128) or NVFP4 as the RMSNorm ops.
 *   weight, bias: device [D] 16-bit, 16-byte aligned, each optional (NULL:
 *   1 / 0).  Other arguments and rules as frt_residual_rmsnorm_fp8 /
 *   frt_residual_rmsnorm_nvfp4.
 *
 * frt_qkv_layernorm_rope_kvcache: "FlashRT kernel fusion", §2.2 second bullet
 * (the Chameleon prefill kernel: LayerNorm(Q) + LayerNorm(K) + rotate-half
 * RoPE in one kernel).  Op (b) with a per-head LayerNorm over hd in place of
 * the RMSNorm:  v' = (v - mean) / sqrt(var + eps) * w[h] + b[h], with
 * per-head affine rows q_w, q_b [Hq, hd] and k_w, k_b [Hkv, hd] (device
 * 16-bit, each optional).  Other arguments, layouts and status bit 0 as
 * frt_qkv_norm_rope_kvcache.
 */
frt_status frt_residual_layernorm_fp8(const void* x, const void* residual_in, void* residual_out, const void* weight,
                                      const void* bias, uint8_t* out_fp8, const float* static_scale,
                                      float* block_scales, int M, int D, float eps, frt_dtype dt, frt_quant qm,
                                      cudaStream_t stream);
frt_status frt_residual_layernorm_nvfp4(const void* x, const void* residual_in, void* residual_out,
                                        const void* weight, const void* bias, uint8_t* out_fp4, uint8_t* out_sf,
                                        const float* global_scale, int M, int D, float eps, frt_dtype dt,
                                        frt_sf_layout sf_layout, cudaStream_t stream);
frt_status frt_qkv_layernorm_rope_kvcache(const void* qkv, const void* q_w, const void* q_b, const void* k_w,
                                          const void* k_b, const float* cos_tab, const float* sin_tab,
                                          const int32_t* positions, void* q_out, void* k_cache, void* v_cache,
                                          int32_t* status, int M, int Hq, int Hkv, int hd, int max_pos,
                                          int capacity, float eps, frt_dtype dt, cudaStream_t stream);

/*
 * NEXT-3: NVFP4 outputs of ops (a) and (c).  The FlashRT port's NVFP4
 * producers "residual_add_rms_norm_to_nvfp4" and "silu_mul_merged_grouped32"
 * (the "5060 Ti" report's per-kernel census and its W4A4 NVFP4 GEMM path).
 * The pages name the format only; the reading is NVFP4:
 *   e2m1 codes (magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6), two per byte with
 *   element 2j in the low nibble of byte j; blocks of 16 consecutive elements
 *   of a row share an unsigned e4m3 scale factor sf; with the per-tensor
 *   global scale gs, y ~ e2m1 * sf * gs.  Decisions in fp32, scaling by
 *   correctly rounded reciprocals (RN = fp32 round to nearest even):
 *     sf   = e4m3(RN(amax_block * RN(1 / RN(6 gs))))  (RNE, saturating to 448)
 *     eff  = RN(sf * gs)
 *     code = e2m1(RN(y * RN(1 / eff)))     (RNE, saturating to 6; 0 when sf = 0)
 *   global_scale must lie in [2^-100, 2^100].
 *
 * frt_residual_rmsnorm_nvfp4: h and y exactly as frt_residual_rmsnorm_fp8
 *   (residual written back); out_fp4 [M, D/2] bytes, 4-byte aligned.
 * frt_gate_act_nvfp4: a exactly as frt_gate_act_fp8; out_fp4 [M, I/2] bytes,
 *   2-byte aligned.
 *   out_sf        device bytes in `sf_layout` (see frt_sf_layout).
 *   global_scale  device fp32[1].
 *   Layout rule: D (I) > 0 and D % 16 == 0 (I % 16 == 0); other arguments
 *   as the FP8 ops.  Unsupported: D > 32768.
 */
frt_status frt_residual_rmsnorm_nvfp4(const void* x, const void* residual_in, void* residual_out, const void* weight,
                                      uint8_t* out_fp4, uint8_t* out_sf, const float* global_scale, int M, int D,
                                      float eps, frt_dtype dt, frt_sf_layout sf_layout, cudaStream_t stream);
frt_status frt_gate_act_nvfp4(const void* gate_up, uint8_t* out_fp4, uint8_t* out_sf, const float* global_scale,
                              int M, int I, frt_act act, frt_dtype dt, frt_sf_layout sf_layout, cudaStream_t stream);

/*
 * NEXT-2: op (b) with the attention's Q preparation and an optional FP8 KV
 * cache.  The "5060 Ti" FlashRT port's optimisation log, step 10: FA2's
 * prepare_q folded into the RoPE kernel (removing 320 launches); "FlashRT
 * kernel fusion", §2.2 for the rest of the op.  The pages name the fusion
 * only; the reading: prepare_q multiplies Q by the attention's softmax scale
 * and may lay Q out head-major, and the KV cache may hold e4m3 codes with a
 * static scale per tensor.
 *
 * Everything as frt_qkv_norm_rope_kvcache, except:
 *   q_out[i, h, :] (token-major) or q_out[h, i, :] (head-major)
 *          = o * q_scale in fp32 (q_scale multiplies the head's norm factor,
 *            or the head before RoPE without a q norm), rounded once to 16
 *            bits;
 *   kv_format E4M3:
 *     k_cache[p, g, :] = e4m3(o / k_scale)  (uint8; o the K head after norm
 *                                           and RoPE, in fp32; the division
 *                                           is a product with RN(1 / k_scale)
 *                                           folded in like q_scale),
 *     v_cache[p, g, :] = e4m3(v / v_scale)  (uint8; the quotient correctly
 *                                           rounded in fp32),
 *     RNE, saturating to +-448.
 *
 *   q_scale      host fp32, finite (1 = no scaling).
 *   q_layout     FRT_Q_TOKEN_MAJOR or FRT_Q_HEAD_MAJOR.
 *   kv_format    FRT_KV_16BIT (caches as op (b)) or FRT_KV_E4M3 (caches
 *                [capacity, Hkv, hd] uint8, 8-byte aligned when hd % 16 == 0,
 *                4-byte aligned when hd % 8 == 0, unaligned otherwise).
 *   kv_scales    device fp32[2] = {k_scale, v_scale}, read with E4M3 only
 *                (may be NULL with 16BIT).
 *   Errors: as op (b); also FRT_ERR_INVALID_ARG for an unknown layout or
 *   format, a non-finite q_scale, or E4M3 without kv_scales.
 */
frt_status frt_qkv_norm_rope_prepq_kvcache(const void* qkv, const void* q_norm_w, const void* k_norm_w,
                                           const float* cos_tab, const float* sin_tab, const int32_t* positions,
                                           void* q_out, void* k_cache, void* v_cache, int32_t* status, int M,
                                           int Hq, int Hkv, int hd, int max_pos, int capacity, float eps,
                                           float q_scale, frt_q_layout q_layout, frt_kv_format kv_format,
                                           const float* kv_scales, frt_dtype dt, cudaStream_t stream);

/*
 * NEXT-1: gated residual + AdaRMSNorm modulation + FP8 quantisation.
 * "FlashRT kernel fusion", §三: the Pi0.5 decoder's cross-layer kernel
 * (gate_res_adarms_fp8_static) fuses gate multiply, residual add, AdaRMSNorm
 * modulation, FP8 quantisation and descale (6 ops -> 1) and runs once per
 * sub-layer per flow step.  The pages give no formula; the reading is the
 * adaptive RMSNorm of flow-matching / diffusion transformers:
 *
 * For row i with condition row c = i / rows_per_cond:
 *   h[i,j]  = residual_in[i,j] + gate[c,j] * x[i,j], the exact value rounded
 *             once to the 16-bit type; written to residual_out.
 *   y[i,j]  = h[i,j] * rstd_i * (1 + scale[c,j]) + shift[c,j],
 *             rstd_i = 1 / sqrt(mean_j(h[i,j]^2) + eps).
 *   out_fp8 = e4m3 of y / s (quant mode as in op (a); block scales over D).
 *             Without scale and shift the arithmetic is op (a)'s (y and the
 *             quotient correctly rounded in fp32); with them y carries a few
 *             fp32 roundings and y / s is a product with 1 / s (folded into
 *             rstd and the shift for a static scale).
 *
 *   x, residual_in, residual_out  device [M, D] 16-bit, 16-byte aligned;
 *                                 residual_out may equal residual_in.
 *   gate, scale, shift            device [ceil(M / rows_per_cond), D] 16-bit,
 *                                 16-byte aligned, or NULL (gate NULL = 1,
 *                                 scale / shift NULL = 0).
 *   out_fp8, static_scale, block_scales  as op (a).
 *   Layout rule: D > 0, D % 8 == 0, rows_per_cond > 0.  Unsupported:
 *   D > 32768.
 */
frt_status frt_gate_residual_adarms_fp8(const void* x, const void* gate, const void* residual_in,
                                        void* residual_out, const void* scale, const void* shift,
                                        uint8_t* out_fp8, const float* static_scale, float* block_scales,
                                        int M, int D, int rows_per_cond, float eps, frt_dtype dt, frt_quant qm,
                                        cudaStream_t stream);

/*
 * Empty kernel used to measure the launch floor that the ops above are graded
 * against (the roofline of a launch-bound op is the larger of its HBM time and
 * this floor).  Launches `grid` blocks of `block` threads that do nothing.
 * Returns FRT_ERR_INVALID_ARG for grid < 1 or block outside [1, 1024].
 */
frt_status frt_noop(int grid, int block, cudaStream_t stream);

/*
 * Dependent-copy probe, the companion of frt_noop: the smallest op that reads
 * what the kernel before it wrote.  `rows` CTAs each copy one row of
 * `row_bytes` bytes from src to dst (device, 16-byte aligned; src == dst is
 * allowed: each 16-byte chunk is read, then written back).  Its time per
 * graph node is the empty-kernel floor plus one dependent load and one store:
 * the floor of any op whose input is its predecessor's output.
 * Returns FRT_ERR_INVALID_ARG for rows < 0, row_bytes <= 0 or not a multiple
 * of 16 (or above 2^30), NULL or misaligned pointers (rows == 0: FRT_OK,
 * nothing launched, pointers not inspected).
 */
frt_status frt_copy_rows(const void* src, void* dst, int rows, int row_bytes, cudaStream_t stream);

/*
 * Programmatic dependent launch (PDL), on by default.  With it on, every
 * kernel of this library is launched with programmatic stream serialisation:
 * the GPU may schedule it while the previous kernel of the same stream is
 * still running (hiding launch latency, e.g. between the nodes of a CUDA
 * graph), and the kernel waits for that previous kernel to complete, with its
 * writes visible (griddepcontrol.wait), before it reads its data inputs (x,
 * residual, qkv, gate_up, the AdaRMSNorm condition rows) or writes anything.
 * Its constant inputs -- norm weights, RoPE tables, positions and the scale
 * inputs (static_scale, kv_scales, global_scale) -- are read before that
 * wait, so they must not be written by the kernel launched just before it on
 * the same stream (no kernel of this library writes them; a host copy or a
 * kernel further back is fine: a kernel is scheduled early only once every
 * CTA of its predecessor has passed its own wait).  Results are identical
 * either way.  The switch is process-wide and read at each launch; changing
 * it while another thread launches affects only later launches.
 */
void frt_set_pdl(int enable);
int frt_get_pdl(void);

/*
 * Bound on the polls of the bulk-copy barrier wait of the QKV ops' large-batch
 * kernel (frt_qkv_norm_rope_kvcache and its NEXT-2 / LayerNorm forms, M >=
 * 592 with 16-byte rows).  That kernel's CTA waits for its token's row to land
 * in shared memory; a wait that runs out of polls sets bit 1 of the op's
 * status word, writes none of the token's outputs, waits once more (with the
 * default bound, whatever this setting) for the copies it issued to land, and
 * returns.  Only a failing device makes the default bound run out; a bound of
 * 0 gives up at once on every token, which lets a test check that path.
 * Process-wide, read at each launch, like frt_set_pdl.
 * Returns FRT_ERR_INVALID_ARG for polls < 0.
 */
#define FRT_DEFAULT_WAIT_POLLS (1 << 22)
frt_status frt_set_wait_polls(int polls);
int frt_get_wait_polls(void);

/* Static, NUL-terminated description of a status value; never NULL. */
const char* frt_status_string(frt_status status);

#ifdef __cplusplus
}
#endif

#endif /* FRT_H_ */
