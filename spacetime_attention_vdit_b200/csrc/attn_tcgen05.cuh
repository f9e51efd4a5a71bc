// attn_tcgen05.cuh - fused flash-style attention forward on the 5th-generation
// tensor cores (tcgen05 + TMEM), TMA-staged Q/K/V tiles.
//
// Computes O = softmax(scale * Q K^T) V per (sequence, head), non-causal: the
// full 3D self-attention of "How AI Generates Video: Inside Sora and Wan2.1 on
// a Real GPU" (section 5: every token attends to every token; section 7: logits
// scaled by 1/sqrt(head_dim)), tiled so that the L x L scores never leave the
// SM ("Video Diffusion Models, in depth", Step 3).  The same kernel runs the
// space pass of divided attention (each frame is a contiguous sequence) and,
// through a strided tensor map, a time pass with long sequences.
//
// One CTA computes two 128-row query tiles (256 rows) of one (sequence, head)
// with three warpgroups:
//   warps 0..3  softmax of query tile 0, warps 4..7 of tile 1, one query row
//               per thread (TMEM lane = row);
//   warp 8      TMA producer: Q tiles once; K_j into a K ring and V_j into a
//               V ring (K is needed one P.V product earlier than V);
//   warp 9      allocates all 512 TMEM columns and issues every UMMA from one
//               thread, in a fixed order: O_i += P_i V_j with P_i read from
//               TMEM (the softmax overwrote tile i's scores with bf16
//               probabilities), then at once S_i = Q_i K_{j+1}^T (smem x smem)
//               into the same columns, for tile 0 and then tile 1;
//   warps 10,11 idle.
// The control warpgroup (8..11) gives registers back after set-up and the
// softmax warpgroups take them (setmaxnreg), so that a softmax thread holds its
// whole row of 128 scores and its packed probabilities without spilling.
// The two tiles ping-pong: while one warpgroup exponentiates its scores the
// tensor core runs the other tile's products.  TMEM columns: S/P of tile i at
// [128 i, 128 i + 128), O of tile i at [256 + 128 i, ...).
//
// Softmax per tile and row: running max m kept unless a new tile raises it by
// more than 8 in log2 units (exact rescaling rule: P stays at most 2^8 and O/l
// is unchanged), the tile's max computed only on the first tile and when the
// tile's sum of P reaches 2^7; P = 2^(s * scale * log2e - m) rounded to bf16,
// one pair in kFmaPairEvery exponentiated on the FMA pipe to unload the MUFU;
// O rescaled in TMEM only when m moved; at the end O / l and the row's
// log-sum-exp are written out.
// kStageO picks how O leaves the SM: false, each thread stores its own row
// with 16-byte stores; true, the rows are staged in the tile's Q buffer and
// sent with TMA stores, which pays off when a CTA sweeps only a few key tiles
// (the host picks true up to 16 key tiles).
//
// Each CTA sweeps the key tiles starting at tile (query block mod tiles), so
// the CTAs of one head, which run together, read different K/V lines from L2
// at any moment instead of all hammering the same ones; the online softmax
// does not depend on the order of the tiles.
#pragma once

#include <math.h>

#include <type_traits>

#include "ptx.cuh"

namespace vdit {

template <int D>
struct AttnCfg {
  static constexpr int BM = 128;                               // query rows per tile
  static constexpr int NQ = 2;                                 // query tiles per CTA
  static constexpr int BN = 128;                               // keys per KV tile
  static constexpr int ROWB = (D * 2 >= 128) ? 128 : D * 2;    // bytes per staged row of one D-block
  static constexpr int DBLK = ROWB / 2;                        // elements per D-block
  static constexpr int NDB = D / DBLK;                         // D-blocks per tile
  static constexpr uint32_t SWZ = ROWB == 128 ? kSwizzle128 : (ROWB == 64 ? kSwizzle64 : kSwizzle32);
  static constexpr int DB_BYTES = BM * ROWB;                   // one D-block of a 128-row tile
  static constexpr int TILE_BYTES = BM * D * 2;
  static constexpr int NK = D >= 128 ? 3 : 4;                  // K ring stages
  static constexpr int NV = D >= 128 ? 2 : (D >= 64 ? 3 : 4);  // V ring stages
  static constexpr int NBARS = 1 + 2 * NK + 2 * NV + 4 * NQ + 1;
  static constexpr int SMEM_BYTES = 1024 + (NQ + NK + NV) * TILE_BYTES + NBARS * 8 + 16;
  static constexpr int THREADS = 384;                          // three warpgroups
  static constexpr int TMA_WARP = 8, MMA_WARP = 9;
  // registers per thread: at launch (what __launch_bounds__(384, 1) allows),
  // then per warpgroup after the split
  static constexpr int REGS_LAUNCH = 168, REGS_SOFTMAX = 216, REGS_CONTROL = 56;
  static_assert(2 * 128 * REGS_SOFTMAX + 128 * REGS_CONTROL <= THREADS * REGS_LAUNCH, "register split");
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t S_COL = 0;                         // tile i: scores / P at 128 i
  static constexpr uint32_t O_COL = 256;                       // tile i: accumulator at 256 + 128 i
  static constexpr uint32_t IDESC_QK = umma_idesc_bf16(BM, BN, 0, 0);  // Q, K both K-major
  static constexpr uint32_t IDESC_PV = umma_idesc_bf16(BM, D, 0, 1);   // P (TMEM) K-major, V MN-major
  static_assert(D % 16 == 0 && D >= 32 && D <= 128, "head_dim");
  static_assert(SMEM_BYTES <= 232448, "shared memory");
};

// Where a (sequence bb, position i) lives among the caller's tokens.
//   kSeq : sequence bb = b*grp + t holds the contiguous tokens [bb*L, bb*L + L)
//          (full attention: grp = 1; space pass: grp = frames per clip).
//   kTime: sequence bb = b*grp + s holds tokens {b*L*grp + i*grp + s} (time pass:
//          grp = sites per frame, L = frames).
enum AttnMode : int { kSeq = 0, kTime = 1 };

struct AttnParams {
  __nv_bfloat16* o;
  float* lse;          // may be null
  int n_seq;           // sequences
  int L;               // query tokens per sequence
  int Lk;              // key tokens per sequence (= L except for cross-attention)
  int heads;
  int grp;             // see AttnMode
  int mode;
  int n_qblocks;       // ceil(L / 256): CTAs per (sequence, head)
  int n_kv;            // ceil(Lk / 128)
  float scale_log2;    // scale * log2(e)
  // Q normalised and rotated in the prologue (attn_fwd_tcgen05_rope_q_kernel only)
  const float2* rope_tab;  // (cos, sin), pair-major: time [pt][Tg], height [ph][Hg], width [pw][Wg]
  const float* wq;         // RMSNorm weight [D], or null (weight 1)
  int rope_tg, rope_hg, rope_wg;  // grid frames, rows and columns
  int rope_pt, rope_ph;    // pairs in the time and height segments (width: the rest)
  int rope_off_h, rope_off_w;  // first table entry of the height and width segments
  int rope_n;              // table entries (at most TILE_BYTES / 8: it is staged in V's second stage)
  int norm;                // 1: RMSNorm over each head's D channels, then the rotation
  float eps, inv_d;        // RMSNorm epsilon, 1/D
};

// Wait sites recorded by the watchdog.
enum : int {
  kSiteQFull = 1, kSiteKFull, kSiteVFull, kSiteKEmpty, kSiteVEmpty, kSiteSFull, kSitePFull, kSiteODone,
  kSiteDrain, kSiteQReady
};

// A wait bounded by time only (used to drain copies and MMAs before exit).
__device__ __forceinline__ void mbar_drain(uint64_t* bar, uint32_t parity) {
  const unsigned long long t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > kWaitLimitNs) { watchdog_trip(kSiteDrain); return; }
  }
}

// 2^x on the FMA pipe: x = n + f with n = rint(x) (the 1.5 * 2^23 rounding
// constant) and |f| <= 1/2; 2^f from a cubic fitted here by relative-error
// least squares on [-1/2, 1/2] (max relative error 7.8e-5, below half a bf16
// ulp); n is added to the exponent field.  x is clamped to at most 8 (so x > 8
// gives 2^8 within the fit's error, which the softmax's sum test relies on: it
// is far above the test's 2^7); below -125 the result is
// 0, like the MUFU's flushed 2^x there, and a masked score (-inf) gives exactly 0.
__device__ __forceinline__ float2 ex2_fma2(float2 x) {
  const float2 xc = make_float2(fminf(fmaxf(x.x, -125.f), 8.f), fminf(fmaxf(x.y, -125.f), 8.f));
  const float2 rnd = make_float2(12582912.f, 12582912.f);
  const float2 t = fadd2(xc, rnd);                                         // rnd + rint(x)
  const float2 f = fadd2(xc, ffma2(t, make_float2(-1.f, -1.f), rnd));     // x - rint(x)
  float2 q = ffma2(make_float2(5.5088737e-2f, 5.5088737e-2f), f, make_float2(0.24260406f, 0.24260406f));
  q = ffma2(q, f, make_float2(0.69327623f, 0.69327623f));
  q = ffma2(q, f, make_float2(0.99992894f, 0.99992894f));
  const float lo = __int_as_float(__float_as_int(q.x) + (__float_as_int(t.x) << 23));
  const float hi = __int_as_float(__float_as_int(q.y) + (__float_as_int(t.y) << 23));
  return make_float2(x.x < -125.f ? 0.f : lo, x.y < -125.f ? 0.f : hi);
}

// One score pair in kFmaPairEvery is exponentiated on the FMA pipe (ex2_fma2),
// the rest on the MUFU: the MUFU alone needs about as many cycles per key tile
// as the tensor core, so a share moved off it shortens the softmax.
#ifndef VDIT_FMA_PAIR_EVERY
#define VDIT_FMA_PAIR_EVERY 32
#endif
constexpr int kFmaPairEvery = VDIT_FMA_PAIR_EVERY;
static_assert(64 % kFmaPairEvery == 0, "pairs per row");

// Packed P columns written per TMEM store (2 keys each).
#ifndef VDIT_P_STORE_COLS
#define VDIT_P_STORE_COLS 8
#endif
constexpr int kPStoreCols = VDIT_P_STORE_COLS;
static_assert(kPStoreCols == 8 || kPStoreCols == 16 || kPStoreCols == 32, "TMEM store width");

// P = 2^(s * scale_log2 - m) for one row's 128 scores, packed to bf16 pairs and
// stored over the row's score columns (pair i of keys 2i, 2i+1 at column i),
// kPStoreCols columns per store so that few packed values are live at once;
// the packed partial sums go to sp.
__device__ __forceinline__ void exp_tile(const uint32_t (&s)[4][32], uint32_t t_s, float2 sc2, float2 nm2,
                                         float2 (&sp)[4]) {
  constexpr int G = kPStoreCols;
#pragma unroll
  for (int g = 0; g < 64 / G; ++g) {
    uint32_t pk[G];
#pragma unroll
    for (int u = 0; u < G; ++u) {
      const int pi = g * G + u;                   // pair of the row
      const int c = pi >> 4, ee = (pi & 15) * 2;
      const float2 x = ffma2(make_float2(__uint_as_float(s[c][ee]), __uint_as_float(s[c][ee + 1])), sc2, nm2);
      const bool on_fma = (pi % kFmaPairEvery) == kFmaPairEvery - 1;
      const float2 pr = on_fma ? ex2_fma2(x) : make_float2(ex2_approx(x.x), ex2_approx(x.y));
      sp[u & 3] = fadd2(sp[u & 3], pr);
      pk[u] = pack_bf16x2(pr.x, pr.y);
    }
    if constexpr (G == 8)
      tmem_st8(t_s + g * G, reinterpret_cast<const uint32_t(&)[8]>(pk));
    else if constexpr (G == 16)
      tmem_st16(t_s + g * G, reinterpret_cast<const uint32_t(&)[16]>(pk));
    else
      tmem_st32(t_s + g * G, reinterpret_cast<const uint32_t(&)[32]>(pk));
  }
}

// Q/K RMSNorm and 3D RoPE of Q in the attention prologue ("How AI Generates
// Video: Inside Sora and Wan2.1 on a Real GPU", section 5, Sub-Layer 1: Q and
// K are RMS-normalised, then rotated by the factorised 3D RoPE of section 4,
// then attend).  While the TMA copy of Q is still landing, the 256 softmax
// threads copy the per-axis (cos, sin) table into V's second ring stage (free
// until the producer's second V load, which waits for both tiles' Q) with
// coalesced loads and meet at a named barrier; fetching each row's 64 pairs
// from global memory instead took several thousand cycles per CTA.  Then one
// softmax thread owns one query row of its tile and rewrites it in place in
// the tile's swizzled shared-memory copy, before the tile's first Q.K^T.  The
// table is pair-major, so the 32 rows of a warp, consecutive tokens, read
// neighbouring entries for each pair (no bank conflicts).  The arithmetic is that of
// the stand-alone passes, operation for operation: the sum of squares of each
// 8-element vector in fused multiply-adds, the vectors' sums added in the
// butterfly order of the per-head norm pass, y = x * rsqrt(mean + eps) * w with
// separately rounded products, the rotation with separately rounded products
// and sums, one rounding to bf16.  So the rotated Q equals the one
// vdit_rope_3d (or vdit_qk_norm_rope_3d with a per-head group) would have
// written, bit for bit.  Returns false if the wait for Q ran out.
template <int D>
__device__ __forceinline__ bool rope_q_rows(const AttnParams& p, unsigned char* tq, float2* tabs, uint64_t* q_full,
                                            uint64_t* q_ready, bool active, int i, int row, int bb, int lane) {
  using C = AttnCfg<D>;
  constexpr int NCH = D / 8;                    // 16-byte chunks of a row
  constexpr int CPB = C::ROWB / 16;             // chunks per staged row of one D-block
  const bool live = active && i < p.L;          // rows past the sequence stay zero
  // every softmax thread takes part, whatever its tile: the barrier counts 256
  for (int x = (int)threadIdx.x; x < p.rope_n; x += 256) tabs[x] = __ldg(p.rope_tab + x);
  // the norm's weights (1 without a weight vector) follow the table
  float* wv = reinterpret_cast<float*>(tabs + p.rope_n);
  if (p.norm)
    for (int x = (int)threadIdx.x; x < D; x += 256) wv[x] = p.wq != nullptr ? __ldg(p.wq + x) : 1.f;
  named_bar_sync(3, 256);
  int bt = 0, bh = 0, bw = 0;
  if (live) {
    // the row's token in its clip (full attention and space pass: contiguous
    // tokens; a long time pass: one site's frames); below 2^31 by the host's
    // size checks
    const uint32_t l = p.mode == kTime ? (uint32_t)i * (uint32_t)p.grp + (uint32_t)(bb % p.grp)
                                       : (uint32_t)(bb % p.grp) * (uint32_t)p.L + (uint32_t)i;
    const uint32_t hw = (uint32_t)p.rope_hg * (uint32_t)p.rope_wg;
    const uint32_t tt = l / hw, rem = l - tt * hw;
    const uint32_t hh = rem / (uint32_t)p.rope_wg, ww = rem - hh * (uint32_t)p.rope_wg;
    // entry of pair pi: base + pi * (its axis's extent)
    bt = (int)tt;
    bh = p.rope_off_h + (int)hh - p.rope_pt * p.rope_hg;
    bw = p.rope_off_w + (int)ww - (p.rope_pt + p.rope_ph) * p.rope_wg;
  }
  bool ok = active;
  if (ok) ok = warp_wait(q_full, 0, kSiteQFull);
  if (ok && live) {
    const int key = C::ROWB == 128 ? (row & 7) : ((row >> 1) & 3);
    auto chunk = [&](int cc) -> uint4* {
      return reinterpret_cast<uint4*>(tq + (cc / CPB) * C::DB_BYTES + row * C::ROWB + (((cc % CPB) ^ key) << 4));
    };
    float nscale = 1.f;
    if (p.norm) {
      float a[NCH];
#pragma unroll
      for (int cc = 0; cc < NCH; ++cc) {
        const uint4 x = *chunk(cc);
        const uint32_t u[4] = {x.x, x.y, x.z, x.w};
        float acc = 0.f;
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const __nv_bfloat162 pr = *reinterpret_cast<const __nv_bfloat162*>(&u[m]);
          const float x0 = __low2float(pr), x1 = __high2float(pr);
          acc = fmaf(x0, x0, acc);
          acc = fmaf(x1, x1, acc);
        }
        a[cc] = acc;
      }
#pragma unroll
      for (int o = NCH / 2; o >= 1; o >>= 1)
#pragma unroll
        for (int k = 0; k < o; ++k) a[k] = a[k] + a[k + o];
      nscale = rsqrtf(fmaf(a[0], p.inv_d, p.eps));
    }
    // Two chunks per iteration: their loads (Q chunks and their pairs' (cos,
    // sin)) are issued before their stores, which the compiler may not move a
    // later shared-memory load above.  The loop is kept rolled: this code runs
    // once per CTA, and fully unrolled (some 1,500 instructions per warp) it
    // ran at a fifth of an instruction per cycle, mostly waiting for
    // instruction fetch.  It is instantiated with and without the norm so
    // that no branch sits inside it.
    auto rotate = [&](auto with_norm) {
      constexpr bool kNorm = decltype(with_norm)::value;
#pragma unroll 1
      for (int c0 = 0; c0 < NCH; c0 += 2) {
        uint4 xv[2];
        float2 cv[2][4];
#pragma unroll
        for (int u = 0; u < 2; ++u) xv[u] = *chunk(c0 + u);
#pragma unroll
        for (int u = 0; u < 2; ++u)
#pragma unroll
          for (int m = 0; m < 4; ++m) {
            const int pi = (c0 + u) * 4 + m;
            cv[u][m] = tabs[pi < p.rope_pt ? bt + pi * p.rope_tg
                                           : (pi < p.rope_pt + p.rope_ph ? bh + pi * p.rope_hg : bw + pi * p.rope_wg)];
          }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int cc = c0 + u;
          uint32_t w[4] = {xv[u].x, xv[u].y, xv[u].z, xv[u].w};
#pragma unroll
          for (int m = 0; m < 4; ++m) {
            const __nv_bfloat162 pr = *reinterpret_cast<const __nv_bfloat162*>(&w[m]);
            float x0 = __low2float(pr), x1 = __high2float(pr);
            if constexpr (kNorm) {
              x0 = __fmul_rn(__fmul_rn(x0, nscale), wv[cc * 8 + 2 * m]);
              x1 = __fmul_rn(__fmul_rn(x1, nscale), wv[cc * 8 + 2 * m + 1]);
            }
            const float2 c = cv[u][m];
            const float re = __fsub_rn(__fmul_rn(x0, c.x), __fmul_rn(x1, c.y));
            const float im = __fadd_rn(__fmul_rn(x0, c.y), __fmul_rn(x1, c.x));
            w[m] = pack_bf16x2(re, im);
          }
          *chunk(cc) = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
    };
    if (p.norm)
      rotate(std::true_type{});
    else
      rotate(std::false_type{});
  }
  // the rewritten rows, and this thread's share of the table copy, are ordered
  // before the tensor core's reads and the TMA's next writes there; then the
  // warp reports (a warp of a tile past the sequence too, since the producer
  // waits for all eight before it overwrites the table; not a warp whose wait
  // for Q ran out, so that nothing reads a Q that may not have landed)
  fence_proxy_async_smem();
  __syncwarp();
  if ((ok || !active) && lane == 0) mbar_arrive(q_ready);
  return ok;
}

template <int D, bool kStageO, bool kRopeQ>
__device__ __forceinline__ void attn_fwd_body(const CUtensorMap& tmQ, const CUtensorMap& tmK,
                                              const CUtensorMap& tmV, const CUtensorMap& tmO,
                                              const AttnParams& p) {
  using C = AttnCfg<D>;
  unsigned char* sQ = smem_base_1024();                            // NQ tiles
  unsigned char* sK = sQ + C::NQ * C::TILE_BYTES;                  // NK tiles
  unsigned char* sV = sK + C::NK * C::TILE_BYTES;                  // NV tiles
  uint64_t* bars = reinterpret_cast<uint64_t*>(sV + C::NV * C::TILE_BYTES);
  uint64_t* q_full = bars;
  uint64_t* k_full = q_full + 1;
  uint64_t* k_empty = k_full + C::NK;
  uint64_t* v_full = k_empty + C::NK;
  uint64_t* v_empty = v_full + C::NV;
  uint64_t* s_full = v_empty + C::NV;      // [NQ]
  uint64_t* p_full = s_full + C::NQ;       // [NQ]
  uint64_t* drain = p_full + C::NQ;        // every UMMA of the CTA has finished
  uint64_t* q_ready = drain + 1;           // [NQ] Q tile rotated in place (kRopeQ)
  uint64_t* o_done = q_ready + C::NQ;      // [NQ] the tile's last P.V (and all before it) finished
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(o_done + C::NQ);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  const int qb = blockIdx.x % p.n_qblocks;
  const int bh = blockIdx.x / p.n_qblocks;
  const int h = bh % p.heads;
  const int bb = bh / p.heads;
  const int q0 = qb * (C::NQ * C::BM);
  const int nq = (q0 + C::BM < p.L) ? 2 : 1;   // query tiles holding rows of the sequence
  const int n = p.n_kv;
  const int j0 = qb % n;                       // first key tile of this CTA's sweep
  // tensor-map coordinates of this sequence: (d, head, site, position, batch)
  const int c_site = p.mode == kTime ? bb % p.grp : 0;
  const int c_batch = p.mode == kTime ? bb / p.grp : bb;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < C::NK; ++s) { mbar_init(&k_full[s], 1); mbar_init(&k_empty[s], 1); }
    for (int s = 0; s < C::NV; ++s) { mbar_init(&v_full[s], 1); mbar_init(&v_empty[s], 1); }
    for (int i = 0; i < C::NQ; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 4);           // one elected lane per softmax warp
      mbar_init(&q_ready[i], 4);
      mbar_init(&o_done[i], 1);
    }
    mbar_init(drain, 1);
    fence_mbar_init();
    // Q and the first K tile, which the first Q.K^T waits for, are requested
    // here, before the CTA-wide set-up (TMEM allocation, the barrier), which
    // their latency then covers; the producer continues from K_1
    mbar_arrive_expect_tx(q_full, nq * C::TILE_BYTES);
    for (int i = 0; i < nq; ++i)
#pragma unroll
      for (int db = 0; db < C::NDB; ++db)
        tma_load_5d(sQ + i * C::TILE_BYTES + db * C::DB_BYTES, &tmQ, q_full, db * C::DBLK, h, c_site,
                    q0 + i * C::BM, c_batch);
    mbar_arrive_expect_tx(&k_full[0], C::TILE_BYTES);
#pragma unroll
    for (int db = 0; db < C::NDB; ++db)
      tma_load_5d(sK + db * C::DB_BYTES, &tmK, &k_full[0], db * C::DBLK, h, c_site, j0 * C::BN, c_batch);
  }
  if (warp == C::MMA_WARP) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // Each warpgroup's branch starts with its register budget, so that the code
  // of each role is compiled for the registers that role holds.
  if (warp >= 8) {
  regs_decrease<C::REGS_CONTROL>();
  if (warp == C::TMA_WARP) {
    // ------------------------------------------------------------------ TMA
    if (lane == 0) {
      tma_prefetch_desc(&tmV);
      int k_issued = 1, v_issued = 0;     // Q and K_0 were requested during set-up
      auto load_k = [&](int j) -> bool {
        const int st = j % C::NK;
        if (j >= C::NK && !mbar_wait(&k_empty[st], ((j / C::NK) - 1) & 1, kSiteKEmpty)) return false;
        mbar_arrive_expect_tx(&k_full[st], C::TILE_BYTES);
#pragma unroll
        for (int db = 0; db < C::NDB; ++db)
          tma_load_5d(sK + st * C::TILE_BYTES + db * C::DB_BYTES, &tmK, &k_full[st], db * C::DBLK, h, c_site,
                      ((j + j0) % n) * C::BN, c_batch);
        k_issued = j + 1;
        return true;
      };
      auto load_v = [&](int j) -> bool {
        const int st = j % C::NV;
        if (j >= C::NV && !mbar_wait(&v_empty[st], ((j / C::NV) - 1) & 1, kSiteVEmpty)) return false;
        mbar_arrive_expect_tx(&v_full[st], C::TILE_BYTES);
#pragma unroll
        for (int db = 0; db < C::NDB; ++db)
          tma_load_5d(sV + st * C::TILE_BYTES + db * C::DB_BYTES, &tmV, &v_full[st], db * C::DBLK, h, c_site,
                      ((j + j0) % n) * C::BN, c_batch);
        v_issued = j + 1;
        return true;
      };
      // K runs one tile ahead of V: K_0, K_1, V_0, K_2, V_1, ...
      bool ok = true;
      for (int j = 0; j < n && ok; ++j) {
        if (j + 1 < n) ok = load_k(j + 1);
        if constexpr (kRopeQ) {
          // V's second stage holds the RoPE table until all eight softmax warps
          // are done with it
          if (j == 1)
            for (int i = 0; i < C::NQ && ok; ++i) ok = mbar_wait(&q_ready[i], 0, kSiteQReady);
        }
        if (ok) ok = load_v(j);
      }
      // No copy may still be landing in shared memory when the CTA exits.
      mbar_drain(q_full, 0);
      for (int j = k_issued - C::NK < 0 ? 0 : k_issued - C::NK; j < k_issued; ++j)
        mbar_drain(&k_full[j % C::NK], (j / C::NK) & 1);
      for (int j = v_issued - C::NV < 0 ? 0 : v_issued - C::NV; j < v_issued; ++j)
        mbar_drain(&v_full[j % C::NV], (j / C::NV) & 1);
    }
  } else if (warp == C::MMA_WARP) {
    // ------------------------------------------------------------------ MMA
    if (lane == 0) {
      const uint32_t sQa = smem_u32(sQ), sKa = smem_u32(sK), sVa = smem_u32(sV);
      constexpr uint32_t SBO = 8 * C::ROWB;       // 8-row core-matrix group stride
      auto qk = [&](int i, int j) {
        const int st = j % C::NK;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk / (C::DBLK / 16)) * C::DB_BYTES + (kk % (C::DBLK / 16)) * 32;
          const uint64_t a = umma_sdesc(sQa + i * C::TILE_BYTES + off, 16, SBO, C::SWZ);
          const uint64_t b = umma_sdesc(sKa + st * C::TILE_BYTES + off, 16, SBO, C::SWZ);
          umma_ss(tmem + C::S_COL + i * C::BN, a, b, C::IDESC_QK, kk > 0 ? 1u : 0u);
        }
        umma_commit(&s_full[i]);
      };
      auto pv = [&](int i, int j) {
        const int st = j % C::NV;
#pragma unroll
        for (int kk = 0; kk < C::BN / 16; ++kk) {
          // A = P_i: 16 keys = 8 TMEM columns of packed bf16 pairs
          // B = V (16 keys x D), MN-major: D-blocks DB_BYTES apart, 8-key groups SBO apart
          const uint64_t b = umma_sdesc(sVa + st * C::TILE_BYTES + kk * 16 * C::ROWB, C::DB_BYTES, SBO, C::SWZ);
          umma_ts(tmem + C::O_COL + i * C::BM, tmem + C::S_COL + i * C::BN + kk * 8, b, C::IDESC_PV,
                  (j > 0 || kk > 0) ? 1u : 0u);
        }
      };
      bool ok;
      if constexpr (kRopeQ) {
        // the first Q.K^T products wait until the softmax warps have rotated
        // Q; both tiles' are then issued back to back, as when Q lands, which
        // starts the two tiles' ping-pong at the offset the loop runs fastest at
        ok = mbar_wait(&k_full[0], 0, kSiteKFull);
        for (int i = 0; i < nq && ok; ++i) ok = mbar_wait(&q_ready[i], 0, kSiteQReady);
        if (ok) {
          tc_fence_after();
          for (int i = 0; i < nq; ++i) qk(i, 0);
          umma_commit(&k_empty[0]);
        }
      } else {
        ok = mbar_wait(q_full, 0, kSiteQFull) && mbar_wait(&k_full[0], 0, kSiteKFull);
        if (ok) {
          tc_fence_after();
          for (int i = 0; i < nq; ++i) qk(i, 0);
          umma_commit(&k_empty[0]);
        }
      }
      // Fixed issue order, the one the two tiles' ping-pong settles into:
      //   O_0 += P_0 V_j, S_0 = Q_0 K_{j+1}^T, O_1 += P_1 V_j, S_1 = Q_1 K_{j+1}^T.
      // QK^T of a tile follows its P.V at once although it overwrites the
      // columns P.V reads: the UMMAs one thread issues execute in issue order
      // (tcgen05 pipelined-instruction ordering), so no wait is needed between
      // them.  The issuing thread sleeps in each barrier wait rather than
      // polling, which would take issue slots from the softmax warp sharing its
      // SM sub-partition.  A K or V stage is released once both tiles have
      // issued the products that read it.
      for (int j = 0; j < n && ok; ++j) {
        for (int i = 0; i < nq; ++i) {
          if (i == 0) ok = mbar_wait(&v_full[j % C::NV], (j / C::NV) & 1, kSiteVFull);
          if (ok) ok = mbar_wait(&p_full[i], j & 1, kSitePFull);
          if (!ok) break;
          tc_fence_after();
          pv(i, j);
          // with few key tiles the epilogue weighs: each tile's starts as soon
          // as its own last P.V is done (long sequences keep the one drain,
          // which measured faster there)
          if (kStageO && j + 1 == n) umma_commit(&o_done[i]);
          if (j + 1 < n) {
            if (i == 0) ok = mbar_wait(&k_full[(j + 1) % C::NK], ((j + 1) / C::NK) & 1, kSiteKFull);
            if (!ok) break;
            qk(i, j + 1);
          }
        }
        if (ok) {
          umma_commit(&v_empty[j % C::NV]);
          if (j + 1 < n) umma_commit(&k_empty[(j + 1) % C::NK]);
        }
      }
      // every UMMA issued above has finished before TMEM is released
      umma_commit(drain);
      mbar_drain(drain, 0);
    }
    __syncwarp();
  }
  } else {
    regs_increase<C::REGS_SOFTMAX>();
    // -------------------------------------------------------------- softmax
    const int tile = warp >> 2;                   // warps 0..3 -> tile 0, 4..7 -> tile 1
    const int quad = warp & 3;                    // TMEM lanes this warp may touch
    const int row = quad * 32 + lane;             // query row within the tile
    const uint32_t tl = tmem + ((uint32_t)(quad * 32) << 16);
    const uint32_t t_s = tl + C::S_COL + tile * C::BN;
    const uint32_t t_o = tl + C::O_COL + tile * C::BM;
    float m_use = -INFINITY;                      // max used for the exponentials (log2 units)
    float l_sum = 0.f;
    bool ok = tile < nq;
    if constexpr (kRopeQ)
      ok = rope_q_rows<D>(p, sQ + tile * C::TILE_BYTES, reinterpret_cast<float2*>(sV + C::TILE_BYTES), q_full,
                          &q_ready[tile], ok, q0 + tile * C::BM + row, row, bb, lane);
    int kt = j0;                                  // key tile of this iteration: (j + j0) mod n, stepped
    for (int j = 0; j < n && ok; ++j, kt = (kt + 1 == n) ? 0 : kt + 1) {
      if (!warp_wait(&s_full[tile], j & 1, kSiteSFull)) { ok = false; break; }
      tc_fence_after();
      uint32_t s[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(t_s + c * 32, s[c]);
      tmem_ld_wait();
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld_fence(s[c]);

      const int valid = p.Lk - kt * C::BN;          // keys of this tile inside the sequence
      if (valid < C::BN) {
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (c * 32 + e >= valid) s[c][e] = __float_as_uint(-INFINITY);
      }
      // the tile's row max, in log2 units
      auto tile_max = [&]() -> float {
        float mp[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};   // four max chains
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int e = 0; e < 32; e += 2)
            mp[(e >> 1) & 3] = fmax3(mp[(e >> 1) & 3], __uint_as_float(s[c][e]), __uint_as_float(s[c][e + 1]));
        return fmaxf(fmax3(mp[0], mp[1], mp[2]), mp[3]) * p.scale_log2;
      };
      // P = 2^(s - m_use) over this tile's own score columns; returns the row's sum
      const float2 sc2 = make_float2(p.scale_log2, p.scale_log2);
      auto exps = [&]() -> float {
        float2 sp[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                        make_float2(0.f, 0.f)};   // four independent packed sum chains
        exp_tile(s, t_s, sc2, make_float2(-m_use, -m_use), sp);
        const float2 s01 = fadd2(fadd2(sp[0], sp[1]), fadd2(sp[2], sp[3]));
        return s01.x + s01.y;
      };
      // The max in use only moves when a tile raises it by more than 8 (log2
      // units; exact: every P stays <= 2^8 and O / l is unchanged).  After the
      // first tile the exponentials are taken against the max in use straight
      // away, and the tile's max is computed only when the tile's sum of P
      // reaches 2^7, which a P above 2^7 implies (the FMA-pipe exponential
      // saturates just below 2^8 for larger arguments, well above 2^7); then,
      // if the max must move, P is taken again.  Once a row's first tiles are
      // in, its scores rarely climb that far, so the max pass leaves the
      // softmax chain.
      float alpha = 1.f;
      if (j == 0) m_use = tile_max();
      float lt = exps();
      if (j > 0 && __any_sync(0xffffffffu, !(lt < 128.f))) {
        const float m_new = tile_max();
        const bool rescale = m_new > m_use + 8.f;
        if (__any_sync(0xffffffffu, rescale)) {   // the stores of P are warp-wide: the warp redoes them
          if (rescale) {
            alpha = ex2_approx(m_use - m_new);
            m_use = m_new;
          }
          tmem_st_wait();       // the first stores of P have landed before they are overwritten
          lt = exps();
          // O follows the max in use (alpha is 1 for the rows whose max stayed)
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tmem_ld32(t_o + c * 32, o);
            tmem_ld_wait();
            tmem_ld_fence(o);
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
            tmem_st32(t_o + c * 32, o);
          }
        }
      }
      l_sum = l_sum * alpha + lt;
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[tile]);
    }

    // ------------------------------------------------------------- epilogue
    if constexpr (!kStageO) {
      // each thread writes its own row of O with 16-byte stores
      if (ok && warp_wait(drain, 0, kSiteODone)) {
        tc_fence_after();
        const int i = q0 + tile * C::BM + row;      // position in the sequence
        const float inv_l = 1.f / l_sum;
        long long token;
        if (p.mode == kTime) {
          const int b = bb / p.grp, sidx = bb % p.grp;
          token = (long long)b * p.L * p.grp + (long long)i * p.grp + sidx;
        } else {
          token = (long long)bb * p.L + i;
        }
        __nv_bfloat16* orow = p.o + (token * p.heads + h) * D;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(t_o + c * 32, o);
          tmem_ld_wait();
          tmem_ld_fence(o);
          if (i < p.L) {
#pragma unroll
            for (int e = 0; e < 32; e += 8) {
              uint4 v;
              v.x = pack_bf16x2(__uint_as_float(o[e + 0]) * inv_l, __uint_as_float(o[e + 1]) * inv_l);
              v.y = pack_bf16x2(__uint_as_float(o[e + 2]) * inv_l, __uint_as_float(o[e + 3]) * inv_l);
              v.z = pack_bf16x2(__uint_as_float(o[e + 4]) * inv_l, __uint_as_float(o[e + 5]) * inv_l);
              v.w = pack_bf16x2(__uint_as_float(o[e + 6]) * inv_l, __uint_as_float(o[e + 7]) * inv_l);
              *reinterpret_cast<uint4*>(orow + c * 32 + e) = v;
            }
          }
        }
        if (p.lse != nullptr && i < p.L) {
          const int b = bb / p.grp, g = bb % p.grp;
          const long long pos = p.mode == kTime ? (long long)i * p.grp + g : (long long)g * p.L + i;
          p.lse[((long long)b * p.heads + h) * ((long long)p.L * p.grp) + pos] =
              (m_use + __log2f(l_sum)) * 0.69314718055994531f;
        }
      }
    } else {
      // O / l is staged in this tile's Q buffer (every UMMA that reads it has
      // finished once o_done fires: UMMAs complete in issue order, and the
      // tile's last Q.K^T precedes its last P.V) in the layout of the
      // Q tensor map; then one thread sends the tile with one TMA store per
      // D-block, rows past the sequence end clipped, so whole 128-byte lines
      // leave the SM instead of a 16-byte piece per row and lane
      bool good = ok;
      if (good) good = warp_wait(&o_done[tile], 0, kSiteODone);
      if (good) {
        tc_fence_after();
        const int i = q0 + tile * C::BM + row;      // position in the sequence
        const float inv_l = 1.f / l_sum;
        unsigned char* stage = sQ + tile * C::TILE_BYTES;
        const int key = C::ROWB == 128 ? (row & 7) : ((row >> 1) & 3);
        constexpr int CPB = C::ROWB / 16;           // 16-byte chunks per staged row
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(t_o + c * 32, o);
          tmem_ld_wait();
          tmem_ld_fence(o);
#pragma unroll
          for (int e = 0; e < 32; e += 8) {
            uint4 v;
            v.x = pack_bf16x2(__uint_as_float(o[e + 0]) * inv_l, __uint_as_float(o[e + 1]) * inv_l);
            v.y = pack_bf16x2(__uint_as_float(o[e + 2]) * inv_l, __uint_as_float(o[e + 3]) * inv_l);
            v.z = pack_bf16x2(__uint_as_float(o[e + 4]) * inv_l, __uint_as_float(o[e + 5]) * inv_l);
            v.w = pack_bf16x2(__uint_as_float(o[e + 6]) * inv_l, __uint_as_float(o[e + 7]) * inv_l);
            const int cc = c * 4 + e / 8;           // 16-byte chunk of the row
            *reinterpret_cast<uint4*>(stage + (cc / CPB) * C::DB_BYTES + row * C::ROWB +
                                      (((cc % CPB) ^ key) << 4)) = v;
          }
        }
        if (p.lse != nullptr && i < p.L) {
          const int b = bb / p.grp, g = bb % p.grp;
          const long long pos = p.mode == kTime ? (long long)i * p.grp + g : (long long)g * p.L + i;
          p.lse[((long long)b * p.heads + h) * ((long long)p.L * p.grp) + pos] =
              (m_use + __log2f(l_sum)) * 0.69314718055994531f;
        }
      }
      // the staged rows become visible to the TMA engine; the tile's four
      // warps meet, and the store goes out only if all four staged their rows
      fence_proxy_async_smem();
      const bool all_good = named_bar_and(1 + tile, 128, good);
      if (all_good && quad == 0 && lane == 0) {
#pragma unroll
        for (int db = 0; db < C::NDB; ++db)
          tma_store_5d(&tmO, sQ + tile * C::TILE_BYTES + db * C::DB_BYTES, db * C::DBLK, h, c_site,
                       q0 + tile * C::BM, c_batch);
        bulk_commit_group();
        bulk_wait_group_read<0>();                  // the buffer is read before the CTA exits
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == C::MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// Full attention, a space pass or a long time pass over Q, K and V as given.
template <int D, bool kStageO>
__global__ void __launch_bounds__(384, 1)
    attn_fwd_tcgen05_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                            const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                            const AttnParams p) {
  attn_fwd_body<D, kStageO, false>(tmQ, tmK, tmV, tmO, p);
}

// The same with Q RMS-normalised (optionally) and rotated by the 3D RoPE in
// the prologue: the caller passes Q as projected, K already normalised and
// rotated.
template <int D, bool kStageO>
__global__ void __launch_bounds__(384, 1)
    attn_fwd_tcgen05_rope_q_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                                   const AttnParams p) {
  attn_fwd_body<D, kStageO, true>(tmQ, tmK, tmV, tmO, p);
}

}  // namespace vdit
