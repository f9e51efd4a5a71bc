/*
 * vdit.h - C ABI of libvdit.so: spacetime self-attention over video-DiT latent
 * tokens on NVIDIA B200 (sm_100a).
 *
 * The hot path the library runs, in the order a video diffusion transformer
 * meets it:
 *
 *   latent clip [N, C, T, H, W]
 *     -> vdit_patchify_3d        cut into (pt, ph, pw) spacetime bricks, one token each
 *        (or vdit_patch_embed_3d: patchify and the Conv3d weight in one pass,
 *         tokens of the model width)
 *     -> (projection to per-head Q, K, V: done by the caller)
 *     -> vdit_rope_3d            factorised 3D rotary positions on Q and K
 *        (or vdit_qk_norm_rope_3d: RMSNorm of Q and K, then the same rotation)
 *     -> vdit_attn_full          full 3D self-attention over all T*H'*W' tokens
 *        (or vdit_attn_full_rope_q: Q normalised and rotated inside the
 *         attention kernel, K by the pass above alone, with the pairs of
 *         vdit_rope_3d_table)
 *        or
 *        vdit_attn_divided_time  attention over the T tokens at each spatial site
 *        vdit_attn_divided_space attention over the H'*W' tokens of each frame
 *     -> vdit_attn_cross         the video tokens attend to the text tokens' keys
 *                                and values (the block's second attention)
 *   and at the end: vdit_unpatchify_3d, tokens back to the latent clip
 *
 * Sources (page title, section):
 *   [towardsai]  "How AI Generates Video: Inside Sora and Wan2.1 on a Real GPU",
 *                sections 4 (spacetime tubes, 3D factorized RoPE), 5 (full 3D
 *                self-attention; "Sub-Layer 2", text cross-attention against
 *                512 prompt tokens) and 7 (the [7800 x 7800] matrix, token
 *                order).
 *   [cheatsheet] "Video and 3D Generation" (aiengineeringfromscratch.com):
 *                "Formulas and numbers" (video tokens, divided attention),
 *                "Tiny video DiT" (Conv3d patchify, time pass then space pass),
 *                "Troubleshooting" (the rope_3d split rule).
 *   [aicassindra] "Video Diffusion Models, in depth": "Step 2: patchify into
 *                spacetime tokens", "Step 3: the diffusion transformer" (tiled
 *                attention whose scores never leave the chip).
 *   [signal3d]   "Video as a 3D signal": "Patches and attention" (full 3-D
 *                against the factorised form).
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Every pointer is a DEVICE pointer owned by the caller.  The library
 *    allocates no memory, frees none and never synchronises; it only enqueues
 *    kernels on `stream` (a cudaStream_t; NULL means the legacy default stream)
 *    and returns.  Calls are asynchronous: data must stay valid until the
 *    stream has run them.
 *  - Token order is time-major, then rows, then columns: token (t', h, w) of a
 *    (Tg, Hg, Wg) grid sits at position t'*Hg*Wg + h*Wg + w [towardsai s.7].
 *  - Q, K, V and O are bfloat16, laid out [B, L, heads, head_dim] (token-major,
 *    heads interleaved: the unpermuted output of a [B, L, heads*head_dim]
 *    projection), contiguous, 16-byte aligned.  Arithmetic is float32.
 *  - head_dim must be 32, 64 or 128 for attention (VDIT_ERR_UNSUPPORTED
 *    otherwise).
 *  - `scale` <= 0 selects 1/sqrt(head_dim) [towardsai s.7].
 *  - `lse` may be NULL.  When given it receives float32 [B, heads, L] natural-log
 *    log-sum-exp of each query row's scaled logits, indexed by the token's own
 *    position in the sequence.
 *  - Host-detectable errors (NULL pointers, bad sizes, misalignment,
 *    unsupported head_dim) return before anything is launched.  A failed
 *    launch returns VDIT_ERR_CUDA.  Faults during execution surface on the
 *    caller's stream, as for any CUDA kernel.
 *  - Failure detection.  Every wait inside a kernel is bounded (2 s).  A wait
 *    that runs out sets a flag word that is ONE per device: every call, stream
 *    and host thread using the device shares it.  While it is set, every later
 *    launch of this library on that device, on any stream, produces no valid
 *    output: the gather and rotation kernels return without writing, and the
 *    tensor-core kernels give up at the first wait that does not complete
 *    within its first 64 polls.  Those calls still return VDIT_OK, because the
 *    host cannot see a device flag without synchronising.  Only
 *    vdit_device_status() reads the flag: it synchronises the whole device,
 *    returns VDIT_ERR_TIMEOUT with the site of the first wait that ran out, and
 *    clears the flag.  A caller that must know that a particular call's output
 *    is valid calls vdit_device_status() after it.  Each call below notes this
 *    as "Watchdog: device-wide".
 */
#ifndef VDIT_H
#define VDIT_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A cudaStream_t, declared without the CUDA headers. */
typedef struct CUstream_st* vdit_stream_t;

/* Status codes returned by every call. */
enum vdit_status {
  VDIT_OK = 0,
  VDIT_ERR_NULL = 1,        /* a required pointer is NULL                       */
  VDIT_ERR_SHAPE = 2,       /* a size is non-positive, inconsistent or too big  */
  VDIT_ERR_ALIGN = 3,       /* a pointer is not 16-byte aligned                 */
  VDIT_ERR_UNSUPPORTED = 4, /* valid input this build does not handle           */
  VDIT_ERR_CUDA = 5,        /* the CUDA runtime reported an error               */
  VDIT_ERR_TIMEOUT = 6      /* a kernel's bounded wait ran out (device status)  */
};

/* Element types of the patchify call. */
enum vdit_dtype { VDIT_F32 = 0, VDIT_BF16 = 1 };

/*
 * vdit_patchify_3d - spacetime patchify [towardsai s.4; cheatsheet "Tiny video
 * DiT": a Conv3d whose stride equals its kernel; aicassindra Step 2].
 *
 *   tokens[n, (t'*Hg + h')*Wg + w', ((c*pt + dt)*ph + dh)*pw + dw]
 *       = latent[n, c, t'*pt + dt, h'*ph + dh, w'*pw + dw]
 *
 * with (Tg, Hg, Wg) = (T/pt, H/ph, W/pw) floored: voxels past the last whole
 * brick are not read.  latent: [N, C, T, H, W] contiguous; tokens:
 * [N, Tg*Hg*Wg, C*pt*ph*pw] contiguous.  dtype VDIT_F32 or VDIT_BF16 for both;
 * values are copied bit for bit.  Pointers need only the element alignment;
 * 16-byte alignment enables vector access.  Errors: VDIT_ERR_NULL,
 * VDIT_ERR_SHAPE (a non-positive size, a grid extent of 0, or more than 2^31
 * tokens), VDIT_ERR_UNSUPPORTED (dtype), VDIT_ERR_CUDA.
 * Watchdog: device-wide (see the conventions above).
 */
int vdit_patchify_3d(const void* latent, void* tokens, int dtype,
                     int N, int C, int T, int H, int W,
                     int pt, int ph, int pw, vdit_stream_t stream);

/*
 * vdit_rope_3d - factorised 3D rotary position embedding [towardsai s.4].
 *
 * Q and K are [B, L, heads, head_dim] bfloat16 with L = Tg*Hg*Wg.  Each head
 * vector is split into a time segment of d_t dims, then d_h, then d_w
 * (d_t + d_h + d_w = head_dim, each even; (44, 42, 42) for head_dim 128).
 * Pair i of a segment of width d (elements 2i and 2i+1 of the segment) turns by
 * the angle pos * theta^(-2i/d), pos being the token's t', h or w on the patch
 * grid:
 *     out[2i]   = x[2i]*cos(a) - x[2i+1]*sin(a)
 *     out[2i+1] = x[2i]*sin(a) + x[2i+1]*cos(a)
 * Angles are formed in float64 and their cosines and sines rounded once to
 * float32, as the page's snippet does; the rotation runs in float32 with each
 * product and sum rounded separately, and the result is rounded to bfloat16
 * (nearest even).  V is not rotated.  q_out/k_out may equal q_in/k_in (in
 * place); otherwise the buffers must not overlap.  q_in and q_out both NULL:
 * K alone is rotated (for vdit_attn_full_rope_q, which rotates Q itself).
 * Errors: VDIT_ERR_NULL (also: one of q_in, q_out NULL but not the other),
 * VDIT_ERR_SHAPE (the split does not add up to head_dim or has an odd or
 * negative part - the page's rope_3d ValueError; non-positive sizes),
 * VDIT_ERR_ALIGN, VDIT_ERR_UNSUPPORTED (head_dim not a multiple of 8),
 * VDIT_ERR_CUDA.
 * Watchdog: device-wide (see the conventions above).
 */
int vdit_rope_3d(const void* q_in, const void* k_in, void* q_out, void* k_out,
                 int B, int Tg, int Hg, int Wg, int heads, int head_dim,
                 int d_t, int d_h, int d_w, float theta, vdit_stream_t stream);

/*
 * vdit_patch_embed_3d - the patch embedding: a Conv3d whose stride equals its
 * kernel [cheatsheet "Tiny video DiT"; towardsai s.4: each 1x2x2 brick of the
 * 16-channel latent becomes one token of the model width], on the tensor cores.
 *
 *   out[n, l, o] = sum_f brick(n, l)[f] * weight[o, f] + bias[o]
 *
 * with brick(n, l) the token's C*pt*ph*pw latent values in vdit_patchify_3d's
 * feature order.  latent: float32 [N, C, T, H, W] (rounded to bfloat16, nearest
 * even, as the tensor-core operand); weight: bfloat16 [dim, C*pt*ph*pw] (the
 * Conv3d weight [dim, C, pt, ph, pw] flattened), 16-byte aligned; bias: NULL
 * or float32 [dim], 16-byte aligned; out: bfloat16 [N, Tg*Hg*Wg, dim], float32
 * accumulation, rounded once.  Extents that do not divide are floored.
 * Errors: VDIT_ERR_NULL, VDIT_ERR_SHAPE, VDIT_ERR_ALIGN, VDIT_ERR_UNSUPPORTED
 * (C*pt*ph*pw other than 64, or dim not a multiple of 256), VDIT_ERR_CUDA.
 * Watchdog: device-wide (see the conventions above).
 */
int vdit_patch_embed_3d(const float* latent, const void* weight, const float* bias, void* out,
                        int N, int C, int T, int H, int W, int pt, int ph, int pw, int dim,
                        vdit_stream_t stream);

/*
 * vdit_unpatchify_3d - the inverse of vdit_patchify_3d: every token's brick is
 * put back, tokens [N, Tg*Hg*Wg, C*pt*ph*pw] -> latent [N, C, Tg*pt, Hg*ph,
 * Wg*pw] (the map from the transformer's last output to the latent clip).  A
 * permutation of values: bit exact, dtype VDIT_F32 or VDIT_BF16.  The buffers
 * must not overlap.
 * Errors: VDIT_ERR_NULL, VDIT_ERR_SHAPE, VDIT_ERR_UNSUPPORTED (dtype, or a token
 * wider than 32 KB), VDIT_ERR_CUDA.
 * Watchdog: device-wide (see the conventions above).
 */
int vdit_unpatchify_3d(const void* tokens, void* latent, int dtype, int N, int C, int Tg, int Hg, int Wg,
                       int pt, int ph, int pw, vdit_stream_t stream);

/*
 * vdit_qk_norm_rope_3d - RMSNorm of Q and K, then the 3D RoPE, in one pass
 * [towardsai s.5, "Sub-Layer 1": the projected Q and K are RMS-normalised, then
 * rotated with the 3D factorized RoPE].
 *
 * Each group of `norm_group` consecutive channels of a token's heads*head_dim
 * channels (head_dim: per head; heads*head_dim: the token's whole vector) is
 *   y = x / sqrt(mean(x^2 over the group) + eps) * w[channel mod norm_group],
 * then rotated exactly as vdit_rope_3d does (same grid, split and theta),
 * float32 throughout and rounded once to bfloat16 (nearest even).
 * wq, wk: NULL (weight 1) or device float32 [norm_group], 16-byte aligned.
 * Layouts, aliasing, the K-only form (q_in and q_out NULL) and the RoPE
 * arguments as for vdit_rope_3d.
 * Errors: VDIT_ERR_NULL, VDIT_ERR_SHAPE (also: norm_group not dividing
 * heads*head_dim, eps negative or not finite), VDIT_ERR_ALIGN,
 * VDIT_ERR_UNSUPPORTED (norm_group not a multiple of 8; a group other than the
 * whole token whose 16-byte vectors, norm_group/8, do not divide 32;
 * heads*head_dim above 8,192; Tg*d_t/2 + Hg*d_h/2 + Wg*d_w/2 above 8,192),
 * VDIT_ERR_CUDA.
 * Watchdog: device-wide (see the conventions above).
 */
int vdit_qk_norm_rope_3d(const void* q_in, const void* k_in, void* q_out, void* k_out,
                         const float* wq, const float* wk, int norm_group, float eps,
                         int B, int Tg, int Hg, int Wg, int heads, int head_dim,
                         int d_t, int d_h, int d_w, float theta, vdit_stream_t stream);

/*
 * vdit_rope_3d_table - the 3D RoPE's (cos, sin) pairs for one token grid
 * [towardsai s.4: the snippet computes its phasors once per shape and keeps
 * them as a cache].
 *
 * table: device float32 [n][2], n = Tg*(d_t/2) + Hg*(d_h/2) + Wg*(d_w/2)
 * (vdit_rope_3d_table_entries), 16-byte aligned, written by the call, pair-major
 * within each axis (neighbouring positions of one pair are neighbouring entries):
 *   entry i*Tg + t'                               time pair i at frame t'
 *   entry Tg*(d_t/2) + i*Hg + h'                  height pair i at row h'
 *   entry Tg*(d_t/2) + Hg*(d_h/2) + i*Wg + w'     width pair i at column w'
 * each holding (cos a, sin a) of a = pos * theta^(-2i/d) for its segment width
 * d, formed in float64 and rounded once to float32: the values vdit_rope_3d
 * rotates with.  The table depends only on the grid, the split and theta; it
 * is an input of vdit_attn_full_rope_q and can be reused by every call on that
 * grid.  Errors: VDIT_ERR_NULL, VDIT_ERR_SHAPE (the split or theta as for
 * vdit_rope_3d; more than 2^31 - 1 entries), VDIT_ERR_ALIGN, VDIT_ERR_CUDA.
 * Watchdog: device-wide (see the conventions above).
 */
int vdit_rope_3d_table(float* table, int Tg, int Hg, int Wg, int head_dim,
                       int d_t, int d_h, int d_w, float theta, vdit_stream_t stream);

/* Entries (float32 pairs) of vdit_rope_3d_table's table, or -1 for a bad grid
 * or split.  Host only; launches nothing. */
long long vdit_rope_3d_table_entries(int Tg, int Hg, int Wg, int head_dim,
                                     int d_t, int d_h, int d_w);

/*
 * vdit_attn_full - full 3D self-attention [towardsai s.5: every token attends
 * to all tokens; aicassindra Step 3: tiled, the L x L scores never reach HBM].
 *
 *   O[b, i, h, :] = sum_j softmax_j(scale * Q[b,i,h,:] . K[b,j,h,:]) V[b, j, h, :]
 *
 * over all L tokens, non-causal, no mask.  q, k, v, o: [B, L, heads, head_dim];
 * lse: NULL or [B, heads, L].  o must not overlap q, k or v.  Runs on the
 * tensor cores (bf16 inputs, float32 accumulation); P is rounded to bfloat16
 * before the P.V product; O is rounded to bfloat16 (nearest even).
 * Errors: VDIT_ERR_NULL, VDIT_ERR_SHAPE, VDIT_ERR_ALIGN, VDIT_ERR_UNSUPPORTED,
 * VDIT_ERR_CUDA.
 * Watchdog: device-wide (see the conventions above).
 */
int vdit_attn_full(const void* q, const void* k, const void* v, void* o, float* lse,
                   int B, int L, int heads, int head_dim, float scale,
                   vdit_stream_t stream);

/*
 * vdit_attn_full_rope_q - full 3D self-attention whose kernel normalises and
 * rotates Q itself [towardsai s.5, "Sub-Layer 1": the projected Q and K are
 * RMS-normalised, rotated with the 3D RoPE of s.4, then attend to each other].
 *
 *   O = vdit_attn_full(q', k, v)   with   q' = rope_3d(norm(q))
 *
 * where norm is the identity (norm_group 0) or the per-head RMSNorm of
 * vdit_qk_norm_rope_3d with norm_group = head_dim and weight wq, and rope_3d
 * is vdit_rope_3d's rotation with the pairs of `rope_table`
 * (vdit_rope_3d_table of the same grid, split and theta).  q' is never
 * written to memory: each CTA rewrites the Q rows it loads, in shared memory,
 * before its first Q.K^T, with the stand-alone passes' arithmetic, so O is the
 * same, bit for bit, as that of the two-step path.  k must already be
 * normalised and rotated (vdit_qk_norm_rope_3d or vdit_rope_3d with q_in and
 * q_out NULL).  A token-wide norm (norm_group = heads*head_dim) needs every head
 * of a token, which one attention CTA does not load: run it with
 * vdit_qk_norm_rope_3d.  q, k, v, o: [B, L, heads, head_dim] with
 * L = Tg*Hg*Wg; lse, numerics and alignment as for vdit_attn_full; wq: NULL
 * (weight 1) or device float32 [head_dim], 16-byte aligned.
 * Errors: VDIT_ERR_NULL, VDIT_ERR_SHAPE (also: the split as for vdit_rope_3d,
 * eps negative or not finite when normalising), VDIT_ERR_ALIGN,
 * VDIT_ERR_UNSUPPORTED (head_dim; norm_group other than 0 or head_dim; a
 * table of n pairs with 8*n + 4*head_dim above 256*head_dim bytes, the
 * shared-memory stage the kernel stages the table and the weights in: 4,032
 * pairs at head_dim 128, more than Tg*22 + (Hg + Wg)*21 for every grid the
 * sources use), VDIT_ERR_CUDA.
 * Watchdog: device-wide (see the conventions above).
 */
int vdit_attn_full_rope_q(const void* q, const void* k, const void* v, void* o, float* lse,
                          int B, int Tg, int Hg, int Wg, int heads, int head_dim, float scale,
                          int d_t, int d_h, int d_w, const float* rope_table,
                          const float* wq, int norm_group, float eps, vdit_stream_t stream);

/*
 * vdit_attn_divided_time - the time pass of divided attention [cheatsheet
 * "Tiny video DiT" and "Divided attention"; signal3d "Patches and attention"].
 *
 * The sequence holds L = T*HW tokens (T frames of HW sites, frame-major).  For
 * each batch b, site s and head h, attention runs over the T tokens
 * {t*HW + s : t < T}; it equals full attention restricted to pairs at the same
 * site.  Buffers as for vdit_attn_full (read and written in place of the
 * tokens; nothing is transposed).  lse: NULL or [B, heads, T*HW].
 * Errors as for vdit_attn_full.
 * Watchdog: device-wide (see the conventions above).
 */
int vdit_attn_divided_time(const void* q, const void* k, const void* v, void* o, float* lse,
                           int B, int T, int HW, int heads, int head_dim, float scale,
                           vdit_stream_t stream);

/*
 * vdit_attn_divided_space - the space pass of divided attention (same sources).
 *
 * For each batch b, frame t and head h, attention runs over the HW tokens of
 * frame t, positions [t*HW, (t+1)*HW); it equals full attention restricted to
 * pairs in the same frame.  Buffers and errors as for
 * vdit_attn_divided_time; lse: NULL or [B, heads, T*HW].
 * Watchdog: device-wide (see the conventions above).
 */
int vdit_attn_divided_space(const void* q, const void* k, const void* v, void* o, float* lse,
                            int B, int T, int HW, int heads, int head_dim, float scale,
                            vdit_stream_t stream);

/*
 * vdit_attn_cross - text cross-attention [towardsai s.5, "Sub-Layer 2": the
 * video tokens supply the queries, the text prompt's tokens the keys and
 * values; aicassindra "Step 3": every block also reads the text embeddings].
 *
 *   O[b, i, h, :] = sum_j softmax_j(scale * Q[b,i,h,:] . K[b,j,h,:]) V[b, j, h, :]
 *
 * with i over the Lq query tokens and j over the Lk key tokens; non-causal, no
 * mask (a caller that pads the prompt passes only the tokens to attend to).
 * q, o: [B, Lq, heads, head_dim]; k, v: [B, Lk, heads, head_dim]; lse: NULL or
 * [B, heads, Lq].  No positions are applied (text tokens carry none).
 * Numerics, alignment and errors as for vdit_attn_full.
 * Watchdog: device-wide (see the conventions above).
 */
int vdit_attn_cross(const void* q, const void* k, const void* v, void* o, float* lse,
                    int B, int Lq, int Lk, int heads, int head_dim, float scale,
                    vdit_stream_t stream);

/* Text for a status code (static storage; never NULL). */
const char* vdit_status_string(int status);

/*
 * vdit_device_status - report and clear the watchdog flags that kernels set
 * when a bounded wait runs out.  Synchronises the current device first (the
 * one call here that does).  *flags (may be NULL) receives the raw bit set:
 * bit 0 any timeout, bits 8.. the wait site.  Returns VDIT_OK when no flag was
 * set, VDIT_ERR_TIMEOUT when one was, VDIT_ERR_CUDA if the device reported an
 * error.
 */
int vdit_device_status(unsigned int* flags);

/*
 * vdit_watchdog_selftest - exercise the failure-detection path.  Enqueues on
 * `stream` one kernel whose single bounded wait (on an mbarrier that nothing
 * arrives on) runs out after the 2-second limit every wait in the library has,
 * and records `site` (1..255) in the device flags exactly as a stalled
 * pipeline would.  Nothing faults and the context stays usable: a following
 * vdit_device_status() returns VDIT_ERR_TIMEOUT with flags bit 0 set and
 * `site` in bits 8..15, and clears them.  While the flag is set, the
 * library's kernels give up at their first wait that does not complete at
 * once (the simplest ones do not start), so their results are not valid: call
 * vdit_device_status() before further work.  Errors: VDIT_ERR_SHAPE (site out
 * of range), VDIT_ERR_CUDA (launch failed).
 */
int vdit_watchdog_selftest(int site, vdit_stream_t stream);

/* Library version, major*10000 + minor*100 + patch. */
int vdit_version(void);

#ifdef __cplusplus
}
#endif

#endif /* VDIT_H */
