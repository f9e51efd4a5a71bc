// patch_embed.cuh - the patch embedding (patchify fused with the product by the
// Conv3d weight, on the 5th-generation tensor cores) and unpatchify.
//
// The patch embedding is a Conv3d whose stride equals its kernel ("Video and 3D
// Generation" cheatsheet, "Tiny video DiT"; "How AI Generates Video: Inside Sora
// and Wan2.1 on a Real GPU", section 4: every 1x2x2 brick of the 16-channel
// latent becomes one token of the model width).  With the Conv3d weight
// flattened to W [dim, F] (F = C*pt*ph*pw, the brick feature order of
// patchify), token l of clip n is  y[n, l, :] = W . brick(n, l) + bias.
// Unpatchify puts each token's brick back: the inverse permutation, which maps
// the transformer's last output to the latent clip.
#pragma once

#include "ptx.cuh"

namespace vdit {

// ---------------------------------------------------------------------------
// Unpatchify
// ---------------------------------------------------------------------------
//
// One CTA per run of WC bricks that share (n, t', h'): their tokens are one
// contiguous span of WC*F elements, copied to shared memory with a padded
// stride (F + 1: the lanes that read one latent row's values from consecutive
// tokens hit different banks), with 16-byte loads when aligned; then one thread
// per (latent row, brick) writes the brick's pw values of that row, so that
// neighbouring lanes store neighbouring addresses.

struct UnpatchifyShape {
  int N, C, pt, ph, pw;
  int Tg, Hg, Wg;   // patch grid
  int F;            // features per token
  int WC;           // bricks per CTA along w'
  int n_wchunks;    // ceil(Wg / WC)
};

constexpr int kUnpatchifyThreads = 256;

template <typename E> struct Pair;
template <> struct Pair<float> { using type = float2; };
template <> struct Pair<__nv_bfloat16> { using type = __nv_bfloat162; };

template <typename E>
__global__ void __launch_bounds__(kUnpatchifyThreads) unpatchify3d_kernel(const E* __restrict__ tokens,
                                                                         E* __restrict__ latent, UnpatchifyShape s,
                                                                         bool vec_in, bool pair_out) {
  E* stage = reinterpret_cast<E*>(dyn_smem);
  if (watchdog_tripped()) return;
  const int T = s.Tg * s.pt, H = s.Hg * s.ph, W = s.Wg * s.pw;
  const long long n_jobs = (long long)s.N * s.Tg * s.Hg * s.n_wchunks;
  const int rs = s.F + 1;                                  // staged token stride
  for (long long job = blockIdx.x; job < n_jobs; job += gridDim.x) {
    const int wc = (int)(job % s.n_wchunks);
    long long r = job / s.n_wchunks;
    const int hq = (int)(r % s.Hg);
    r /= s.Hg;
    const int tq = (int)(r % s.Tg);
    const int n = (int)(r / s.Tg);
    const int w0 = wc * s.WC;
    const int nb = min(s.WC, s.Wg - w0);
    const E* src = tokens + ((((long long)n * s.Tg + tq) * s.Hg + hq) * s.Wg + w0) * s.F;
    __syncthreads();
    if (vec_in) {                                           // 16-byte loads, 16 / sizeof(E) elements each
      constexpr int V = 16 / sizeof(E);
      const int n4 = nb * s.F / V;
      for (int e4 = threadIdx.x; e4 < n4; e4 += blockDim.x) {
        const uint4 u = reinterpret_cast<const uint4*>(src)[e4];
        const E* ue = reinterpret_cast<const E*>(&u);
        const int e = e4 * V, b = e / s.F, f = e - b * s.F;   // F is a multiple of V: one token
#pragma unroll
        for (int m = 0; m < V; ++m) stage[b * rs + f + m] = ue[m];
      }
    } else {
      for (int e = threadIdx.x; e < nb * s.F; e += blockDim.x) {
        const int b = e / s.F, f = e - b * s.F;
        stage[b * rs + f] = src[e];
      }
    }
    __syncthreads();
    // one warp per latent row (c, dt, dh), one lane per brick: the brick's pw
    // values of the row, which are consecutive features of the token;
    // neighbouring lanes take neighbouring bricks, so the stores are contiguous
    const int nrows = s.C * s.pt * s.ph;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
    for (int row = warp; row < nrows; row += nwarps) {   // row = (c, dt, dh)
      const int dh = row % s.ph, cdt = row / s.ph;
      const int dt = cdt % s.pt, c = cdt / s.pt;
      const int f0 = ((c * s.pt + dt) * s.ph + dh) * s.pw;
      E* drow = latent + (((long long)n * s.C + c) * T + tq * s.pt + dt) * ((long long)H * W) +
                (long long)(hq * s.ph + dh) * W + (long long)w0 * s.pw;
      for (int b = lane; b < nb; b += 32) {
        const E* sp = stage + b * rs + f0;
        E* dst = drow + (long long)b * s.pw;
        if (pair_out) {                                   // pw == 2: one 2-element store
          typename Pair<E>::type v;
          v.x = sp[0];
          v.y = sp[1];
          *reinterpret_cast<typename Pair<E>::type*>(dst) = v;
        } else {
          for (int dw = 0; dw < s.pw; ++dw) dst[dw] = sp[dw];
        }
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Patch embedding on the tensor cores
// ---------------------------------------------------------------------------
//
// Tokens are taken 128 at a time (a token tile, M = 128) and the model width
// 256 at a time (an N tile); K = F = 64 features (one 128-byte swizzle row of
// bf16).  CTAs are persistent over token tiles.  Per CTA:
//   warp 0      TMA producer: the weight's N tiles [256 x 64] bf16 (K-major,
//               128-byte swizzle) into a 3-stage ring, in the order the MMA
//               thread consumes them (every N tile for each token tile; the
//               192 KB weight stays in L2);
//   warp 1      allocates 512 TMEM columns (two 256-column accumulators) and
//               issues the UMMAs: 4 x (M128, N256, K16) per N tile;
//   warps 6..9  build the token tile's A operand: thread r gathers token r's
//               64 brick features from the float32 latent, rounds them to
//               bf16 and writes the 128-byte row in the swizzled layout (two
//               A buffers, so the next tile is gathered during this one's
//               products);
//   warps 2..5  epilogue: accumulator + bias, rounded to bf16; one thread per
//               token row (TMEM lane = row).  Each warp writes its 32 rows of a
//               64-column box into a staging buffer of its own (128-byte
//               swizzle) and lane 0 sends it out with a TMA store, so the
//               stores are whole lines and the warps never wait on each other.
// Every wait is bounded by the watchdog; copies and UMMAs are drained before
// the CTA exits.

constexpr int kEmbBM = 128, kEmbBN = 256, kEmbK = 64;
constexpr int kEmbNW = 3;                                  // weight ring stages
constexpr int kEmbThreads = 320;
constexpr int kEmbATile = kEmbBM * kEmbK * 2;              // 16 KB
constexpr int kEmbWTile = kEmbBN * kEmbK * 2;              // 32 KB
constexpr int kEmbOutBox = 64;                              // output columns per TMA store box
constexpr int kEmbStage = 32 * kEmbOutBox * 2;             // one warp's box: 32 rows x 128 bytes
constexpr int kEmbNStage = 4;                              // staging boxes per warp
constexpr int kEmbSmem = 1024 + 2 * kEmbATile + kEmbNW * kEmbWTile + 4 * kEmbNStage * kEmbStage + 256 + kEmbK * 4;
constexpr uint32_t kEmbIdesc = umma_idesc_bf16(kEmbBM, kEmbBN, 0, 0);

struct EmbedParams {
  const float* latent;
  const float* bias;         // [dim] or null
  __nv_bfloat16* out;        // [N, L, dim]
  int C, T, H, W, pt, ph, pw, Tg, Hg, Wg;
  long long ntok;            // N * L
  int dim;                   // model width, a multiple of 256
  int n_mt;                  // token tiles
  int group_nt;              // N tiles per work item
  int n_groups;              // work items per token tile
  int n_items;               // n_mt * n_groups
};

enum : int { kSiteEmbA = 40, kSiteEmbW, kSiteEmbAcc, kSiteEmbDrain };

__global__ void __launch_bounds__(kEmbThreads, 1)
    patch_embed_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmOut,
                       const EmbedParams p) {
  unsigned char* sA = smem_base_1024();                                 // 2 A buffers
  unsigned char* sW = sA + 2 * kEmbATile;                                // weight ring
  unsigned char* sOut = sW + kEmbNW * kEmbWTile;                       // [epilogue warp][kEmbNStage] boxes
  uint64_t* bars = reinterpret_cast<uint64_t*>(sOut + 4 * kEmbNStage * kEmbStage);
  uint64_t* a_full = bars;            // [2] the gather warps filled the buffer
  uint64_t* a_empty = a_full + 2;     // [2] the buffer's UMMAs finished
  uint64_t* w_full = a_empty + 2;     // [kEmbNW]
  uint64_t* w_empty = w_full + kEmbNW;
  uint64_t* acc_full = w_empty + kEmbNW;   // [2]
  uint64_t* acc_empty = acc_full + 2;      // [2]
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  int* f_off = reinterpret_cast<int*>(bars + 32);                        // latent offset of feature f in a brick

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_nt = p.dim / kEmbBN;
  // Work item w = (token tile w / n_groups, N tiles [g G, g G + G) with g = w mod
  // n_groups): CTA c takes items c, c + gridDim.x, ...  Splitting a token tile's
  // N tiles over several items keeps the last wave of CTAs short.
  const int n_my = (int)blockIdx.x < p.n_items ? (p.n_items - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
  auto item_w = [&](int lt) { return (int)blockIdx.x + lt * (int)gridDim.x; };
  auto item_tm = [&](int lt) { return item_w(lt) / p.n_groups; };
  auto item_nt0 = [&](int lt) { return (item_w(lt) % p.n_groups) * p.group_nt; };
  auto item_nn = [&](int lt) { return min(p.group_nt, n_nt - item_nt0(lt)); };
  const long long plane = (long long)p.H * p.W;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&a_full[i], 4);
      mbar_init(&a_empty[i], 1);
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 4);
    }
    for (int i = 0; i < kEmbNW; ++i) { mbar_init(&w_full[i], 1); mbar_init(&w_empty[i], 1); }
    mbar_init(drain, 1);
    fence_mbar_init();
  }
  for (int f = threadIdx.x; f < kEmbK; f += blockDim.x) {
    const int dw = f % p.pw, r1 = f / p.pw;
    const int dh = r1 % p.ph, r2 = r1 / p.ph;
    const int dt = r2 % p.pt, c = r2 / p.pt;
    f_off[f] = (int)(((long long)c * p.T + dt) * plane + (long long)dh * p.W + dw);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA
    if (lane == 0) {
      tma_prefetch_desc(&tmW);
      int issued = 0;
      bool ok = true;
      for (int lt = 0; lt < n_my && ok; ++lt) {
        const int nt0 = item_nt0(lt), nn = item_nn(lt);
        for (int j = 0; j < nn; ++j) {
          const int st = issued, s = st % kEmbNW;
          if (st >= kEmbNW && !mbar_wait(&w_empty[s], ((st / kEmbNW) - 1) & 1, kSiteEmbW)) { ok = false; break; }
          mbar_arrive_expect_tx(&w_full[s], kEmbWTile);
          tma_load_2d(sW + s * kEmbWTile, &tmW, &w_full[s], 0, (nt0 + j) * kEmbBN);
          ++issued;
        }
      }
      for (int st = issued - kEmbNW < 0 ? 0 : issued - kEmbNW; st < issued; ++st)
        mbar_drain_site(&w_full[st % kEmbNW], (st / kEmbNW) & 1, kSiteEmbDrain);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA
    if (lane == 0) {
      const uint32_t sAa = smem_u32(sA), sWa = smem_u32(sW);
      bool ok = true;
      int st = 0;                                       // N tiles done by this CTA
      for (int lt = 0; lt < n_my && ok; ++lt) {
        const int ab = lt & 1;
        if (!mbar_wait(&a_full[ab], (lt >> 1) & 1, kSiteEmbA)) { ok = false; break; }
        const int nn = item_nn(lt);
        for (int j = 0; j < nn && ok; ++j, ++st) {
          const int s = st % kEmbNW, ac = st & 1;
          if (!mbar_wait(&w_full[s], (st / kEmbNW) & 1, kSiteEmbW) ||
              (st >= 2 && !mbar_wait(&acc_empty[ac], ((st >> 1) - 1) & 1, kSiteEmbAcc))) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < kEmbK / 16; ++kk) {
            const uint64_t a = umma_sdesc(sAa + ab * kEmbATile + kk * 32, 16, 1024, kSwizzle128);
            const uint64_t b = umma_sdesc(sWa + s * kEmbWTile + kk * 32, 16, 1024, kSwizzle128);
            umma_ss(tmem + ac * kEmbBN, a, b, kEmbIdesc, kk > 0 ? 1u : 0u);
          }
          umma_commit(&w_empty[s]);
          umma_commit(&acc_full[ac]);
        }
        if (ok) umma_commit(&a_empty[ab]);
      }
      umma_commit(drain);
      mbar_drain_site(drain, 0, kSiteEmbDrain);
    }
    __syncwarp();
  } else if (warp >= 6) {
    // ------------------------------------------------------------- gather
    const int r = (warp - 6) * 32 + lane;               // token row of the tile
    for (int lt = 0; lt < n_my; ++lt) {
      const int ab = lt & 1;
      if (lt >= 2 && !warp_wait(&a_empty[ab], ((lt >> 1) - 1) & 1, kSiteEmbA)) break;
      const long long tok = (long long)item_tm(lt) * kEmbBM + r;
      unsigned char* row = sA + ab * kEmbATile + r * 128;
      if (tok < p.ntok) {
        long long q = tok;
        const int wq = (int)(q % p.Wg);
        q /= p.Wg;
        const int hq = (int)(q % p.Hg);
        q /= p.Hg;
        const int tq = (int)(q % p.Tg);
        const int n = (int)(q / p.Tg);
        const float* origin = p.latent + ((long long)n * p.C * p.T + (long long)tq * p.pt) * plane +
                              (long long)hq * p.ph * p.W + (long long)wq * p.pw;
#pragma unroll
        for (int j = 0; j < kEmbK / 8; ++j) {             // 16-byte chunk j: features 8j .. 8j+7
          uint4 v;
          v.x = pack_bf16x2(__ldg(origin + f_off[8 * j + 0]), __ldg(origin + f_off[8 * j + 1]));
          v.y = pack_bf16x2(__ldg(origin + f_off[8 * j + 2]), __ldg(origin + f_off[8 * j + 3]));
          v.z = pack_bf16x2(__ldg(origin + f_off[8 * j + 4]), __ldg(origin + f_off[8 * j + 5]));
          v.w = pack_bf16x2(__ldg(origin + f_off[8 * j + 6]), __ldg(origin + f_off[8 * j + 7]));
          *reinterpret_cast<uint4*>(row + ((j ^ (r & 7)) << 4)) = v;
        }
      } else {
#pragma unroll
        for (int j = 0; j < kEmbK / 8; ++j) *reinterpret_cast<uint4*>(row + ((j ^ (r & 7)) << 4)) = make_uint4(0, 0, 0, 0);
      }
      fence_proxy_async_smem();                         // the tensor core reads what the threads wrote
      __syncwarp();
      if (lane == 0) mbar_arrive(&a_full[ab]);
    }
  } else {
    // ----------------------------------------------------------- epilogue
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const uint32_t tl = tmem + ((uint32_t)(quad * 32) << 16);
    unsigned char* my_stage = sOut + quad * kEmbNStage * kEmbStage;
    int boxes = 0;                                      // boxes this warp has sent
    int st = 0;                                         // N tiles done by this CTA
    for (int lt = 0; lt < n_my; ++lt) {
      const long long tile0 = (long long)item_tm(lt) * kEmbBM;
      const int nt0 = item_nt0(lt), nn = item_nn(lt);
      bool ok = true;
      for (int j = 0; j < nn; ++j, ++st) {
        const int nt = nt0 + j, ac = st & 1;
        if (!warp_wait(&acc_full[ac], (st >> 1) & 1, kSiteEmbAcc)) { ok = false; break; }
        tc_fence_after();
#pragma unroll 1
        for (int bx = 0; bx < kEmbBN / kEmbOutBox; ++bx, ++boxes) {
          unsigned char* box = my_stage + (boxes % kEmbNStage) * kEmbStage;
          if (boxes >= kEmbNStage) {                    // the TMA store that used this buffer has read it
            if (lane == 0) bulk_wait_group_read<kEmbNStage - 1>();
            __syncwarp();
          }
#pragma unroll
          for (int h = 0; h < kEmbOutBox / 32; ++h) {
            uint32_t o[32];
            tmem_ld32(tl + ac * kEmbBN + bx * kEmbOutBox + h * 32, o);
            tmem_ld_wait();
            tmem_ld_fence(o);
            const int col = nt * kEmbBN + bx * kEmbOutBox + h * 32;
#pragma unroll
            for (int e = 0; e < 32; e += 8) {
              float b8[8];
              if (p.bias != nullptr) {
                const float4 b0 = __ldg(reinterpret_cast<const float4*>(p.bias + col + e));
                const float4 b1 = __ldg(reinterpret_cast<const float4*>(p.bias + col + e + 4));
                b8[0] = b0.x; b8[1] = b0.y; b8[2] = b0.z; b8[3] = b0.w;
                b8[4] = b1.x; b8[5] = b1.y; b8[6] = b1.z; b8[7] = b1.w;
              } else {
#pragma unroll
                for (int m = 0; m < 8; ++m) b8[m] = 0.f;
              }
              uint4 v;
              v.x = pack_bf16x2(__uint_as_float(o[e + 0]) + b8[0], __uint_as_float(o[e + 1]) + b8[1]);
              v.y = pack_bf16x2(__uint_as_float(o[e + 2]) + b8[2], __uint_as_float(o[e + 3]) + b8[3]);
              v.z = pack_bf16x2(__uint_as_float(o[e + 4]) + b8[4], __uint_as_float(o[e + 5]) + b8[5]);
              v.w = pack_bf16x2(__uint_as_float(o[e + 6]) + b8[6], __uint_as_float(o[e + 7]) + b8[7]);
              const int j = h * 4 + e / 8;              // 16-byte chunk of the 128-byte row
              *reinterpret_cast<uint4*>(box + lane * 128 + ((j ^ (lane & 7)) << 4)) = v;
            }
          }
          fence_proxy_async_smem();                     // the TMA engine reads what the lanes wrote
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&tmOut, box, nt * kEmbBN + bx * kEmbOutBox, (int)(tile0 + quad * 32));
            bulk_commit_group();
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[ac]);
      }
      if (!ok) break;
    }
    if (lane == 0) bulk_wait_group_all();               // every store has landed before the CTA exits
    (void)r;
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace vdit
