// patchify_rope.cuh - the two bandwidth-bound steps of the path.
//
// Spacetime patchify ("How AI Generates Video: Inside Sora and Wan2.1 on a Real
// GPU", section 4; "Video and 3D Generation" cheatsheet, "Tiny video DiT": a
// Conv3d whose stride equals its kernel) is a pure permutation of the latent
// clip.  Factorised 3D RoPE (same article, section 4) rotates adjacent pairs of
// every Q and K head vector by angles set by the token's (t', h, w).
#pragma once

#include "ptx.cuh"

namespace vdit {

// ---------------------------------------------------------------------------
// Patchify
// ---------------------------------------------------------------------------
//
// One CTA owns a run of WC bricks that share (n, t', h') - consecutive tokens,
// so its output is one contiguous span of WC*F elements (F = C*pt*ph*pw).  The
// CTA first copies the C*pt*ph latent rows those bricks cover (each a
// contiguous run of WC*pw elements along W) into shared memory, one warp per
// row with 16-byte loads (four in flight per lane) when the row is aligned;
// then it writes the output span with 16-byte stores, each gathering VEC
// consecutive features from the staged rows through a per-CTA table of staged
// offsets.  Staged rows are an odd number of elements apart, so the lanes that
// gather one brick's channels (one per staged row) fall in different banks.
// Unaligned shapes take the same path one element at a time.

struct PatchifyShape {
  int N, C, T, H, W, pt, ph, pw;
  int Tg, Hg, Wg;   // patch grid (floored)
  int F;            // features per token
  int WC;           // bricks per CTA along w'
  int n_wchunks;    // ceil(Wg / WC)
};

constexpr int kPatchifyThreads = 256;
// The (1, 2, 2) float32 path runs small CTAs, many per SM, so that one CTA's
// loads overlap another's stores; each job keeps a whole latent row, since
// shorter contiguous runs cost more than the lost occupancy.
constexpr int kPatchify122Threads = 128;
constexpr int kPatchify122CtasPerSm = 32;

template <typename E>
__global__ void __launch_bounds__(kPatchifyThreads) patchify3d_kernel(const E* __restrict__ latent,
                                                                      E* __restrict__ tokens, PatchifyShape s) {
  constexpr int VEC = 16 / sizeof(E);             // elements per 16-byte vector
  // dynamic shared memory: F staged-row offsets (int), then the staged rows
  int* src_off = reinterpret_cast<int*>(dyn_smem);
  E* rows = reinterpret_cast<E*>(dyn_smem + ((s.F * sizeof(int) + 15) & ~size_t(15)));
  if (watchdog_tripped()) return;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
  const int rowlen = s.WC * s.pw + ((s.WC * s.pw) % 2 == 0 ? 1 : 0);   // staged row stride (odd)
  const int nrows = s.C * s.pt * s.ph;
  // feature f = ((c*pt + dt)*ph + dh)*pw + dw  reads staged row (c*pt + dt)*ph + dh at dw
  for (int f = threadIdx.x; f < s.F; f += blockDim.x) src_off[f] = (f / s.pw) * rowlen + f % s.pw;
  // 16-byte paths: every staged row starts 16-byte aligned in global and shared
  // memory, and every output span does too
  const bool vec_in = (s.W % VEC) == 0 && ((s.WC * s.pw) % VEC) == 0 &&
                      (reinterpret_cast<uintptr_t>(latent) & 15) == 0;
  const bool vec_out = (s.F % VEC) == 0 && (reinterpret_cast<uintptr_t>(tokens) & 15) == 0;

  const long long n_jobs = (long long)s.N * s.Tg * s.Hg * s.n_wchunks;
  for (long long job = blockIdx.x; job < n_jobs; job += gridDim.x) {
    const int wc = (int)(job % s.n_wchunks);
    long long r = job / s.n_wchunks;
    const int hq = (int)(r % s.Hg);
    r /= s.Hg;
    const int tq = (int)(r % s.Tg);
    const int n = (int)(r / s.Tg);
    const int w0 = wc * s.WC;
    const int nb = min(s.WC, s.Wg - w0);          // bricks in this chunk
    const int len = nb * s.pw;                    // valid elements per staged row

    __syncthreads();                              // previous job's rows consumed; table written
    // stage latent rows (c, dt, dh): one warp per row
    for (int row = warp; row < nrows; row += nwarps) {
      const int dh = row % s.ph;
      const int cdt = row / s.ph;
      const int dt = cdt % s.pt;
      const int c = cdt / s.pt;
      const E* src = latent + ((((long long)n * s.C + c) * s.T + (tq * s.pt + dt)) * s.H + (hq * s.ph + dh)) *
                                  (long long)s.W + (long long)w0 * s.pw;
      E* dst = rows + row * rowlen;
      if (vec_in) {
        const int nv = len / VEC;                 // whole 16-byte vectors of the row
        const uint4* sv = reinterpret_cast<const uint4*>(src);
        for (int x = lane; x < nv; x += 128) {
          union { uint4 u; E e[VEC]; } t[4];
#pragma unroll
          for (int u = 0; u < 4; ++u)
            if (x + 32 * u < nv) t[u].u = __ldg(sv + x + 32 * u);
#pragma unroll
          for (int u = 0; u < 4; ++u)
            if (x + 32 * u < nv) {
#pragma unroll
              for (int k = 0; k < VEC; ++k) dst[(x + 32 * u) * VEC + k] = t[u].e[k];
            }
        }
        for (int x = nv * VEC + lane; x < len; x += 32) dst[x] = src[x];   // tail shorter than a vector
      } else {
        for (int x = lane; x < len; x += 32) dst[x] = src[x];
      }
    }
    __syncthreads();

    // write the contiguous output span of nb tokens
    E* out = tokens + (((long long)n * s.Tg + tq) * s.Hg * s.Wg + (long long)hq * s.Wg + w0) * s.F;
    if (vec_out) {
      const int gpb = s.F / VEC;                  // vectors per brick
      for (int g = threadIdx.x; g < nb * gpb; g += blockDim.x) {
        const int b = g / gpb;
        const int f0 = (g - b * gpb) * VEC;
        const E* from = rows + b * s.pw;
        union { uint4 u; E e[VEC]; } v;
#pragma unroll
        for (int k = 0; k < VEC; ++k) v.e[k] = from[src_off[f0 + k]];
        reinterpret_cast<uint4*>(out)[g] = v.u;
      }
    } else {
      for (int b = warp; b < nb; b += nwarps) {
        const E* from = rows + b * s.pw;
        E* to = out + (long long)b * s.F;
        for (int f = lane; f < s.F; f += 32) to[f] = from[src_off[f]];
      }
    }
  }
}

// The pages' own patch, (1, 2, 2), on float32: each output float4 is one channel
// of one brick, {row(c, dh = 0)[2b], [2b + 1], row(c, 1)[2b], [2b + 1]}, i.e. two
// float2 reads from two staged rows - no offset table.  Staged rows are
// 2*WC + 2 floats apart (8-byte aligned, 2 words mod 32 banks), which keeps the
// float2 staging stores and the float2 gathers at or near the two-wavefront
// minimum of a 256-byte warp access.  Output float4 stores are coalesced.
__global__ void __launch_bounds__(kPatchify122Threads) patchify122_f32_kernel(const float* __restrict__ latent,
                                                                           float* __restrict__ tokens,
                                                                           PatchifyShape s) {
  float* rows = reinterpret_cast<float*>(dyn_smem);
  if (watchdog_tripped()) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
  const int rs = 2 * s.WC + 2;                    // staged row stride (floats)
  const int nrows = 2 * s.C;                      // (c, dh)
  const long long plane = (long long)s.H * s.W;
  const long long n_jobs = (long long)s.N * s.Tg * s.Hg * s.n_wchunks;
  for (long long job = blockIdx.x; job < n_jobs; job += gridDim.x) {
    const int wc = (int)(job % s.n_wchunks);
    long long r = job / s.n_wchunks;
    const int hq = (int)(r % s.Hg);
    r /= s.Hg;
    const int tq = (int)(r % s.Tg);
    const int n = (int)(r / s.Tg);
    const int w0 = wc * s.WC;
    const int nb = min(s.WC, s.Wg - w0);
    const int len = 2 * nb;                       // floats of each staged row
    __syncthreads();
    for (int row = warp; row < nrows; row += nwarps) {
      const int c = row >> 1, dh = row & 1;
      const float* src = latent + (((long long)n * s.C + c) * s.T + tq) * plane + (long long)(2 * hq + dh) * s.W +
                         2LL * w0;
      float* dst = rows + row * rs;
      const int n4 = len >> 2;                    // 16-byte vectors (src is 16-byte aligned, see launcher)
      const float4* sv = reinterpret_cast<const float4*>(src);
      for (int x = lane; x < n4; x += 128) {
        float4 t[4];
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if (x + 32 * u < n4) t[u] = __ldg(sv + x + 32 * u);
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if (x + 32 * u < n4) {
            float2* d = reinterpret_cast<float2*>(dst + 4 * (x + 32 * u));
            d[0] = make_float2(t[u].x, t[u].y);
            d[1] = make_float2(t[u].z, t[u].w);
          }
      }
      for (int x = 4 * n4 + lane; x < len; x += 32) dst[x] = src[x];
    }
    __syncthreads();
    float4* out = reinterpret_cast<float4*>(tokens + (((long long)n * s.Tg + tq) * s.Hg * s.Wg +
                                                      (long long)hq * s.Wg + w0) * s.F);
    for (int g = threadIdx.x; g < nb * s.C; g += blockDim.x) {
      const int b = g / s.C, c = g - b * s.C;
      const float2 a = *reinterpret_cast<const float2*>(rows + (2 * c) * rs + 2 * b);
      const float2 d = *reinterpret_cast<const float2*>(rows + (2 * c + 1) * rs + 2 * b);
      out[g] = make_float4(a.x, a.y, d.x, d.y);
    }
  }
}

// ---------------------------------------------------------------------------
// 3D RoPE
// ---------------------------------------------------------------------------
//
// A CTA handles kRopeTokens tokens per iteration (grid-stride over tokens).
// For those tokens it first builds the (cos, sin) of every pair in shared
// memory: angle = pos * inv_freq in float64, cos and sin in float64, each
// rounded once to float32 (the snippet's complex64 cache).  inv_freq[p] =
// 1 / theta^(2i/d) for pair i of its axis segment is built once per CTA.  Then
// all heads of Q and K for those tokens stream through 16-byte vectors (four
// pairs each); each pair is rotated with separately rounded float32 products
// and sums and stored as bfloat16, round to nearest even.  With one tensor
// (K only, passed in the Q slots) the same loop covers that tensor alone.

constexpr int kRopeThreads = 256;
constexpr int kRopeTokens = 4;
constexpr int kRopeMaxPairs = 128;  // head_dim <= 256
constexpr int kRopeBatch = 4;       // 16-byte loads in flight per thread

struct RopeShape {
  long long ntok;     // B * L
  int L, Hg, Wg;      // tokens per sequence, grid rows and columns
  int heads, D;       // head count, head width
  int pt_end, ph_end; // pair index where the h segment starts, and the w segment
  int d_t, d_h, d_w;
  int ntens;          // 2: Q and K; 1: one tensor (K), passed in the Q slots
};

// (cos, sin) of pos * theta^(-2i/d) for pair i of a segment of width d: the
// angle formed in float64, cos and sin rounded once to float32 (the snippet's
// complex64 cache).
__device__ __forceinline__ float2 rope_phasor(int pos, int i, int d, double theta) {
  double sn, cn;
  sincos((double)pos * (1.0 / pow(theta, (double)(2 * i) / (double)d)), &sn, &cn);
  return make_float2((float)cn, (float)sn);
}

// Entry x of the position-major per-axis table: time [Tg][d_t/2], then height
// [Hg][d_h/2] from off_h, then width [Wg][d_w/2] from off_w.
__device__ __forceinline__ float2 rope_axis_entry(int x, int off_h, int off_w, int d_t, int d_h, int d_w,
                                                  double theta) {
  const int pt = d_t / 2, ph = d_h / 2, pw = d_w / 2;
  int pos, i, d;
  if (x < off_h) { pos = x / pt; i = x - pos * pt; d = d_t; }
  else if (x < off_w) { pos = (x - off_h) / ph; i = x - off_h - pos * ph; d = d_h; }
  else { pos = (x - off_w) / pw; i = x - off_w - pos * pw; d = d_w; }
  return rope_phasor(pos, i, d, theta);
}

// The whole per-axis table in global memory, pair-major (time [d_t/2][Tg],
// then height [d_h/2][Hg], then width [d_w/2][Wg]), for kernels that look the
// pairs of consecutive tokens up together (the attention kernel that rotates
// Q itself): for one pair, neighbouring positions are neighbouring entries.
__global__ void rope3d_table_kernel(float2* tab, int Tg, int Hg, int Wg, int d_t, int d_h, int d_w,
                                    double theta) {
  if (watchdog_tripped()) return;
  const int off_h = Tg * (d_t / 2), off_w = off_h + Hg * (d_h / 2), n = off_w + Wg * (d_w / 2);
  for (int x = blockIdx.x * blockDim.x + threadIdx.x; x < n; x += gridDim.x * blockDim.x) {
    int pos, i, d;
    if (x < off_h) { i = x / Tg; pos = x - i * Tg; d = d_t; }
    else if (x < off_w) { i = (x - off_h) / Hg; pos = x - off_h - i * Hg; d = d_h; }
    else { i = (x - off_w) / Wg; pos = x - off_w - i * Wg; d = d_w; }
    tab[x] = rope_phasor(pos, i, d, theta);
  }
}

__global__ void __launch_bounds__(kRopeThreads) rope3d_kernel(const __nv_bfloat16* q_in, const __nv_bfloat16* k_in,
                                                              __nv_bfloat16* q_out, __nv_bfloat16* k_out,
                                                              RopeShape s, double theta) {
  __shared__ double inv_freq[kRopeMaxPairs];
  __shared__ float2 cs[kRopeTokens][kRopeMaxPairs];
  if (watchdog_tripped()) return;

  const int P = s.D / 2;
  for (int p = threadIdx.x; p < P; p += blockDim.x) {
    int i, d;
    if (p < s.pt_end) { i = p; d = s.d_t; }
    else if (p < s.ph_end) { i = p - s.pt_end; d = s.d_h; }
    else { i = p - s.ph_end; d = s.d_w; }
    inv_freq[p] = 1.0 / pow(theta, (double)(2 * i) / (double)d);
  }
  __syncthreads();

  const int vec_per_head = s.D / 8;                      // 16-byte vectors (4 pairs) per head
  const int vec_per_tok = s.heads * vec_per_head;        // per tensor
  for (long long tok0 = (long long)blockIdx.x * kRopeTokens; tok0 < s.ntok;
       tok0 += (long long)gridDim.x * kRopeTokens) {
    const int nt = (int)min((long long)kRopeTokens, s.ntok - tok0);
    for (int e = threadIdx.x; e < nt * P; e += blockDim.x) {
      const int j = e / P, p = e - j * P;
      const int l = (int)((tok0 + j) % s.L);
      int pos;
      if (p < s.pt_end) pos = l / (s.Hg * s.Wg);
      else if (p < s.ph_end) pos = (l / s.Wg) % s.Hg;
      else pos = l % s.Wg;
      double sn, cn;
      sincos((double)pos * inv_freq[p], &sn, &cn);
      cs[j][p] = make_float2((float)cn, (float)sn);
    }
    __syncthreads();

    // Each thread keeps kRopeBatch 16-byte loads in flight before rotating them.
    // Every vector is read and written by the same thread, so in-place use is safe.
    const int nvec = nt * vec_per_tok;                   // per tensor
    for (int e0 = threadIdx.x; e0 < s.ntens * nvec; e0 += blockDim.x * kRopeBatch) {
      uint4 v[kRopeBatch];
#pragma unroll
      for (int u = 0; u < kRopeBatch; ++u) {
        const int e = e0 + u * blockDim.x;
        if (e < s.ntens * nvec) {
          const int which = e >= nvec;                   // 0: Q, 1: K
          const int ee = which ? e - nvec : e;
          const long long off = tok0 * (long long)vec_per_tok + ee;
          v[u] = *(reinterpret_cast<const uint4*>(which ? k_in : q_in) + off);
        }
      }
#pragma unroll
      for (int u = 0; u < kRopeBatch; ++u) {
        const int e = e0 + u * blockDim.x;
        if (e < s.ntens * nvec) {
          const int which = e >= nvec;
          const int ee = which ? e - nvec : e;
          const int j = ee / vec_per_tok;
          const int p0 = ((ee - j * vec_per_tok) % vec_per_head) * 4;
          uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            __nv_bfloat162 pr = *reinterpret_cast<__nv_bfloat162*>(&w[t]);
            const float x0 = __low2float(pr), x1 = __high2float(pr);
            const float2 c = cs[j][p0 + t];
            const float re = __fsub_rn(__fmul_rn(x0, c.x), __fmul_rn(x1, c.y));
            const float im = __fadd_rn(__fmul_rn(x0, c.y), __fmul_rn(x1, c.x));
            w[t] = pack_bf16x2(re, im);
          }
          const long long off = tok0 * (long long)vec_per_tok + ee;
          *(reinterpret_cast<uint4*>(which ? k_out : q_out) + off) = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
    }
    __syncthreads();
  }
}

// ---------------------------------------------------------------------------
// Q/K RMSNorm fused with the 3D RoPE
// ---------------------------------------------------------------------------
//
// "How AI Generates Video: Inside Sora and Wan2.1 on a Real GPU", section 5
// (Sub-Layer 1): the projected Q and K are RMS-normalised, then rotated.  One
// HBM pass does both.  A CTA walks its tokens (blockIdx.x + k * gridDim.x);
// thread 0 streams each token's Q and K rows (heads*D bf16 each) into a ring
// of kNormStages shared-memory stages with bulk copies, kNormStages tokens
// ahead, so that several tokens per CTA are in flight.  For the token at hand
// threads 0..127 take Q and 128..255 K, thread t the 16-byte vectors t,
// t + 128, ...; each group of `group` channels is summed in float32 (a
// segmented shuffle reduction when a group's vectors sit in consecutive lanes of
// one warp, or warp sums added over the tensor's four warps when the group is
// the whole token); then y = x * rsqrt(mean + eps) * weight[channel mod group],
// rotated like rope3d_kernel (separately rounded float32 products), rounded
// once to bfloat16 and stored.  A CTA-wide barrier at the end of each token
// frees its stage for the copy kNormStages tokens later.  The (cos, sin) of
// every pair at every position of its axis (Tg x d_t/2 + Hg x d_h/2 + Wg x
// d_w/2 entries) are built once per CTA in shared memory, after the ring, so
// that a token's rotation is a table lookup.  With one tensor (K only) just
// K's rows are copied and threads 0..127 only take part in the barriers.

constexpr int kNormThreads = 256;
constexpr int kNormStages = 4;
constexpr int kNormVecs = 8;        // vectors per thread: heads * head_dim <= 128 * 8 * 8 = 8,192
constexpr int kSiteNormFull = 30, kSiteNormDrain = 31;   // watchdog wait sites
constexpr int kNormMaxTable = 8192;  // (cos, sin) table entries: Tg*d_t/2 + Hg*d_h/2 + Wg*d_w/2

template <bool kWide>   // the group is the token's whole heads*D vector
__global__ void __launch_bounds__(kNormThreads) qk_norm_rope3d_kernel(
    const __nv_bfloat16* q_in, const __nv_bfloat16* k_in, __nv_bfloat16* q_out, __nv_bfloat16* k_out,
    const float* __restrict__ wq, const float* __restrict__ wk, RopeShape s, int group, float eps, double theta) {
  __shared__ float wsum[2][4];                          // [tensor][warp]: sums of squares
  __shared__ float2 cs[2][kRopeMaxPairs];              // the token's pairs, by token parity
  __shared__ __align__(8) uint64_t full[kNormStages];
  if (__syncthreads_or(watchdog_tripped())) return;    // all threads of the CTA decide alike

  const int vec_per_head = s.D / 8;
  const int nv = s.heads * vec_per_head;                // vectors per token and tensor
  uint4* ring = reinterpret_cast<uint4*>(dyn_smem);    // [stage][Q row, K row] of nv vectors each
  // per-axis tables: time [Tg][d_t/2], then height [Hg][d_h/2], then width [Wg][d_w/2]
  float2* tab = reinterpret_cast<float2*>(ring + (size_t)kNormStages * 2 * nv);
  const int pt = s.d_t / 2, ph = s.d_h / 2, pw = s.d_w / 2;
  const int Tg = (int)(s.L / ((long long)s.Hg * s.Wg));
  const int off_h = Tg * pt, off_w = off_h + s.Hg * ph, n_tab = off_w + s.Wg * pw;
  for (int x = threadIdx.x; x < n_tab; x += blockDim.x)
    tab[x] = rope_axis_entry(x, off_h, off_w, s.d_t, s.d_h, s.d_w, theta);
  if (threadIdx.x == 0) {
    for (int st = 0; st < kNormStages; ++st) mbar_init(&full[st], 1);
    fence_mbar_init();
  }
  __syncthreads();

  const uint32_t row_bytes = (uint32_t)nv * 16u;
  const long long n_my = (s.ntok - 1 - blockIdx.x) / gridDim.x + 1;   // grid <= ntok
  auto issue = [&](long long k) {                       // thread 0: token k of this CTA into its stage
    const int st = (int)(k % kNormStages);
    const long long tok = blockIdx.x + k * gridDim.x;
    mbar_arrive_expect_tx(&full[st], (uint32_t)s.ntens * row_bytes);
    if (s.ntens == 2) bulk_load(ring + (size_t)st * 2 * nv, q_in + tok * nv * 8, row_bytes, &full[st]);
    bulk_load(ring + (size_t)st * 2 * nv + nv, k_in + tok * nv * 8, row_bytes, &full[st]);
  };
  long long issued = n_my < kNormStages ? n_my : kNormStages;
  if (threadIdx.x == 0)
    for (long long k = 0; k < issued; ++k) issue(k);

  const int which = threadIdx.x >> 7;                   // 0: Q, 1: K
  const bool active = which == 1 || s.ntens == 2;       // K only: the Q threads idle between barriers
  const int t = threadIdx.x & 127;
  const int lane = threadIdx.x & 31, wt = t >> 5;       // warp within the tensor's four
  const int gv = group / 8;                             // vectors per group
  const float inv_group = 1.f / (float)group;
  const float* w = which ? wk : wq;
  long long k = 0;
  for (; k < n_my; ++k) {
    const long long tok = blockIdx.x + k * gridDim.x;
    const int l = (int)(tok % s.L);
    const int par = (int)(k & 1);
    if (threadIdx.x < (unsigned)(pt + ph + pw)) {       // the token's row of pairs, from the axis tables
      const int pp = threadIdx.x;
      float2 c;
      if (pp < pt) c = tab[(l / (s.Hg * s.Wg)) * pt + pp];
      else if (pp < pt + ph) c = tab[off_h + ((l / s.Wg) % s.Hg) * ph + (pp - pt)];
      else c = tab[off_w + (l % s.Wg) * pw + (pp - pt - ph)];
      cs[par][pp] = c;
    }
    const int st = (int)(k % kNormStages);
    const bool okw = mbar_wait(&full[st], (uint32_t)((k / kNormStages) & 1), kSiteNormFull);
    if (!__syncthreads_and(okw)) break;                 // also publishes cs[par]
    const uint4* sv = ring + (size_t)st * 2 * nv + (size_t)which * nv;
    uint4 v[kNormVecs];
#pragma unroll
    for (int r = 0; r < kNormVecs; ++r) {
      const int e = t + 128 * r;
      v[r] = (e < nv && active) ? sv[e] : make_uint4(0u, 0u, 0u, 0u);
    }
    auto vec_sq = [&](const uint4& x) -> float {
      const uint32_t u[4] = {x.x, x.y, x.z, x.w};
      float a = 0.f;
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const __nv_bfloat162 pr = *reinterpret_cast<const __nv_bfloat162*>(&u[m]);
        const float x0 = __low2float(pr), x1 = __high2float(pr);
        a = fmaf(x0, x0, a);
        a = fmaf(x1, x1, a);
      }
      return a;
    };
    float tok_sq = 0.f;
    if (kWide) {
#pragma unroll
      for (int r = 0; r < kNormVecs; ++r) tok_sq += vec_sq(v[r]);
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) tok_sq += __shfl_xor_sync(0xffffffffu, tok_sq, o);
      if (lane == 0) wsum[which][wt] = tok_sq;
      __syncthreads();
      tok_sq = (wsum[which][0] + wsum[which][1]) + (wsum[which][2] + wsum[which][3]);
    }
    uint4* dst = reinterpret_cast<uint4*>(which ? k_out : q_out) + tok * nv;
#pragma unroll
    for (int r = 0; r < kNormVecs; ++r) {
      float sq = tok_sq;
      if (!kWide) {                                     // the group's gv vectors: gv consecutive lanes
        sq = vec_sq(v[r]);
        for (int o = gv >> 1; o >= 1; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
      }
      const int e = t + 128 * r;
      if (e < nv && active) {
        const float scale = rsqrtf(fmaf(sq, inv_group, eps));
        const int c0 = (e * 8) % group;                 // channel of the vector's first element in its group
        float wv[8];
        if (w != nullptr) {
          const float4 w0 = __ldg(reinterpret_cast<const float4*>(w + c0));
          const float4 w1 = __ldg(reinterpret_cast<const float4*>(w + c0 + 4));
          wv[0] = w0.x; wv[1] = w0.y; wv[2] = w0.z; wv[3] = w0.w;
          wv[4] = w1.x; wv[5] = w1.y; wv[6] = w1.z; wv[7] = w1.w;
        } else {
#pragma unroll
          for (int m = 0; m < 8; ++m) wv[m] = 1.f;
        }
        const int p0 = (e % vec_per_head) * 4;
        uint32_t u[4] = {v[r].x, v[r].y, v[r].z, v[r].w};
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const __nv_bfloat162 pr = *reinterpret_cast<const __nv_bfloat162*>(&u[m]);
          const float x0 = __fmul_rn(__fmul_rn(__low2float(pr), scale), wv[2 * m]);
          const float x1 = __fmul_rn(__fmul_rn(__high2float(pr), scale), wv[2 * m + 1]);
          const float2 c = cs[par][p0 + m];
          const float re = __fsub_rn(__fmul_rn(x0, c.x), __fmul_rn(x1, c.y));
          const float im = __fadd_rn(__fmul_rn(x0, c.y), __fmul_rn(x1, c.x));
          u[m] = pack_bf16x2(re, im);
        }
        dst[e] = make_uint4(u[0], u[1], u[2], u[3]);
      }
    }
    __syncthreads();                                    // the stage (and wsum) is free
    if (threadIdx.x == 0 && issued < n_my) issue(issued++);
  }
  // No copy may still be landing in shared memory when the CTA exits (only
  // when a wait above ran out can tokens k .. issued-1 still be in flight).
  if (threadIdx.x == 0)
    for (long long k2 = k; k2 < issued; ++k2)
      mbar_drain_site(&full[k2 % kNormStages], (uint32_t)((k2 / kNormStages) & 1), kSiteNormDrain);
}

}  // namespace vdit
