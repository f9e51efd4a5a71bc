// vdit_api.cu - the C ABI of libvdit.so (declared in include/vdit.h).
//
// Host side, apart from the watchdog's self-check kernel: argument checks that
// return before any launch, tensor-map encoding for the TMA loads and stores,
// grid sizing, and the launches themselves.  One translation unit holds every
// kernel so that the watchdog flag is a single device symbol.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "vdit.h"
#include "attn_tcgen05.cuh"
#include "attn_time_short.cuh"
#include "patchify_rope.cuh"
#include "patch_embed.cuh"

namespace {

using namespace vdit;

constexpr int kMaxDevices = 64;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int last_launch_status() { return cudaGetLastError() == cudaSuccess ? VDIT_OK : VDIT_ERR_CUDA; }

int sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) != cudaSuccess) return n;
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

// Set a kernel's dynamic shared-memory limit once per device.
template <typename K>
bool ensure_smem(K kernel, int bytes, bool (&done)[kMaxDevices]) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
  if (!done[dev]) {
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
      return false;
    done[dev] = true;
  }
  return true;
}

// ---------------------------------------------------------------------------
// Tensor maps
// ---------------------------------------------------------------------------

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 5-D view {head_dim, heads, sites, positions, batches} of a bf16 [.., heads, D]
// token array; box {DBLK, 1, 1, box_rows, 1}.  Rows outside the positions extent
// read as zero.
bool make_qkv_map(CUtensorMap* map, const void* base, int D, int heads, long long sites, long long positions,
                  long long batches, long long site_stride_el, long long pos_stride_el, long long batch_stride_el,
                  int box_rows = 128) {
  EncodeTiledFn enc = encode_tiled();
  if (enc == nullptr) return false;
  const int rowb = D * 2 >= 128 ? 128 : D * 2;
  const cuuint64_t dims[5] = {(cuuint64_t)D, (cuuint64_t)heads, (cuuint64_t)sites, (cuuint64_t)positions,
                              (cuuint64_t)batches};
  const cuuint64_t strides[4] = {(cuuint64_t)D * 2, (cuuint64_t)site_stride_el * 2, (cuuint64_t)pos_stride_el * 2,
                                 (cuuint64_t)batch_stride_el * 2};
  const cuuint32_t box[5] = {(cuuint32_t)(rowb / 2), 1, 1, (cuuint32_t)box_rows, 1};
  const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  const CUtensorMapSwizzle sw = rowb == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                : rowb == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                             : CU_TENSOR_MAP_SWIZZLE_32B;
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D view {cols, rows} of a row-major bf16 matrix (cols a multiple of 8);
// box {box_cols, box_rows}, 128-byte swizzle when a box row is 128 bytes.
bool make_2d_map(CUtensorMap* map, const void* base, long long cols, long long rows, int box_cols, int box_rows) {
  EncodeTiledFn enc = encode_tiled();
  if (enc == nullptr) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  const cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, box_cols * 2 == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ---------------------------------------------------------------------------
// Attention launches
// ---------------------------------------------------------------------------

// Key tiles (of 128 keys) up to which the kernel stages O for TMA stores.
constexpr int kStagedOMaxKeyTiles = 16;

// `rope`: null, or the RoPE fields of AttnParams for the kernel that rotates Q
// in its prologue.
template <int D>
int launch_tcgen05(const void* q, const void* k, const void* v, void* o, float* lse, int mode, int n_seq, int L,
                   int Lk, int grp, int heads, float scale, cudaStream_t stream, const AttnParams* rope = nullptr) {
  using C = AttnCfg<D>;
  static bool smem_row[kMaxDevices] = {}, smem_staged[kMaxDevices] = {};
  static bool smem_row_r[kMaxDevices] = {}, smem_staged_r[kMaxDevices] = {};
  static std::mutex mu;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (!ensure_smem(attn_fwd_tcgen05_kernel<D, false>, C::SMEM_BYTES, smem_row) ||
        !ensure_smem(attn_fwd_tcgen05_kernel<D, true>, C::SMEM_BYTES, smem_staged) ||
        !ensure_smem(attn_fwd_tcgen05_rope_q_kernel<D, false>, C::SMEM_BYTES, smem_row_r) ||
        !ensure_smem(attn_fwd_tcgen05_rope_q_kernel<D, true>, C::SMEM_BYTES, smem_staged_r))
      return VDIT_ERR_CUDA;
  }
  // geometry of the 5-D view
  long long sites, positions, batches, site_stride, pos_stride, batch_stride;
  const long long tok = (long long)heads * D;      // elements per token
  if (mode == kTime) {            // sequence = one site across frames
    sites = grp;
    positions = L;
    batches = n_seq / grp;
    site_stride = tok;
    pos_stride = tok * grp;
    batch_stride = tok * grp * L;
  } else {                        // sequence = a contiguous run of L tokens
    sites = 1;
    positions = L;
    batches = n_seq;
    site_stride = tok;
    pos_stride = tok;
    batch_stride = tok * L;
  }
  // keys and values: the same view, with Lk positions per sequence when they
  // come from another token array (cross-attention; kSeq only)
  const long long k_positions = mode == kTime ? positions : Lk;
  const long long k_batch_stride = mode == kTime ? batch_stride : tok * Lk;
  // O is written through a map of the same shape as Q's (the kernel's TMA stores)
  CUtensorMap mq, mk, mv, mo;
  if (!make_qkv_map(&mq, q, D, heads, sites, positions, batches, site_stride, pos_stride, batch_stride) ||
      !make_qkv_map(&mk, k, D, heads, sites, k_positions, batches, site_stride, pos_stride, k_batch_stride) ||
      !make_qkv_map(&mv, v, D, heads, sites, k_positions, batches, site_stride, pos_stride, k_batch_stride) ||
      !make_qkv_map(&mo, o, D, heads, sites, positions, batches, site_stride, pos_stride, batch_stride))
    return VDIT_ERR_CUDA;
  AttnParams p = rope != nullptr ? *rope : AttnParams{};
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.n_seq = n_seq;
  p.L = L;
  p.Lk = mode == kTime ? L : Lk;
  p.heads = heads;
  p.grp = grp;
  p.mode = mode;
  p.n_qblocks = (L + C::NQ * C::BM - 1) / (C::NQ * C::BM);
  p.n_kv = (p.Lk + C::BN - 1) / C::BN;
  p.scale_log2 = scale * 1.4426950408889634f;
  const long long grid = (long long)n_seq * heads * p.n_qblocks;
  if (grid > 0x7fffffffLL) return VDIT_ERR_SHAPE;
  // Short key sequences (cross-attention to a prompt, the space pass at 480p)
  // give each CTA few key tiles, so its epilogue weighs: O goes out staged in
  // shared memory by TMA stores.  Long ones keep the per-row stores, whose
  // variant of the kernel runs its key-tile loop faster.
  const bool staged = p.n_kv <= kStagedOMaxKeyTiles;
  const unsigned g = (unsigned)grid;
  if (rope != nullptr) {
    if (staged)
      attn_fwd_tcgen05_rope_q_kernel<D, true><<<g, C::THREADS, C::SMEM_BYTES, stream>>>(mq, mk, mv, mo, p);
    else
      attn_fwd_tcgen05_rope_q_kernel<D, false><<<g, C::THREADS, C::SMEM_BYTES, stream>>>(mq, mk, mv, mo, p);
  } else if (staged) {
    attn_fwd_tcgen05_kernel<D, true><<<g, C::THREADS, C::SMEM_BYTES, stream>>>(mq, mk, mv, mo, p);
  } else {
    attn_fwd_tcgen05_kernel<D, false><<<g, C::THREADS, C::SMEM_BYTES, stream>>>(mq, mk, mv, mo, p);
  }
  return last_launch_status();
}

int dispatch_tcgen05(int D, const void* q, const void* k, const void* v, void* o, float* lse, int mode, int n_seq,
                     int L, int Lk, int grp, int heads, float scale, cudaStream_t stream,
                     const AttnParams* rope = nullptr) {
  switch (D) {
    case 32: return launch_tcgen05<32>(q, k, v, o, lse, mode, n_seq, L, Lk, grp, heads, scale, stream, rope);
    case 64: return launch_tcgen05<64>(q, k, v, o, lse, mode, n_seq, L, Lk, grp, heads, scale, stream, rope);
    case 128: return launch_tcgen05<128>(q, k, v, o, lse, mode, n_seq, L, Lk, grp, heads, scale, stream, rope);
    default: return VDIT_ERR_UNSUPPORTED;
  }
}

// Checks shared by the RoPE calls: grid, split and theta.
int check_rope_shape(int Tg, int Hg, int Wg, int head_dim, int d_t, int d_h, int d_w, float theta) {
  if (Tg <= 0 || Hg <= 0 || Wg <= 0 || head_dim <= 0) return VDIT_ERR_SHAPE;
  if (d_t < 0 || d_h < 0 || d_w < 0 || (d_t | d_h | d_w) & 1 || d_t + d_h + d_w != head_dim) return VDIT_ERR_SHAPE;
  if (!(theta > 0.f) || !std::isfinite(theta)) return VDIT_ERR_SHAPE;
  if ((long long)Tg * Hg * Wg > 0x7fffffffLL) return VDIT_ERR_SHAPE;
  return VDIT_OK;
}

long long rope_table_entries(int Tg, int Hg, int Wg, int d_t, int d_h, int d_w) {
  return (long long)Tg * (d_t / 2) + (long long)Hg * (d_h / 2) + (long long)Wg * (d_w / 2);
}

template <int D, int TB>
int launch_time_short(const void* q, const void* k, const void* v, const TimeParams& p, cudaStream_t stream) {
  using C = TimeCfg<D, TB>;
  static bool smem_done[kMaxDevices] = {};
  static std::mutex mu;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (!ensure_smem(attn_time_short_kernel<D, TB>, C::SMEM_BYTES, smem_done)) return VDIT_ERR_CUDA;
  }
  // view {D, heads, sites, frames, batch}; one box = one site's TB frames of one head
  const long long tok = (long long)p.heads * D;
  CUtensorMap mq, mk, mv;
  const long long site_st = tok, frame_st = tok * p.HW, batch_st = tok * p.HW * p.T;
  if (!make_qkv_map(&mq, q, D, p.heads, p.HW, p.T, p.B, site_st, frame_st, batch_st, TB) ||
      !make_qkv_map(&mk, k, D, p.heads, p.HW, p.T, p.B, site_st, frame_st, batch_st, TB) ||
      !make_qkv_map(&mv, v, D, p.heads, p.HW, p.T, p.B, site_st, frame_st, batch_st, TB))
    return VDIT_ERR_CUDA;
  const long long units = (long long)p.B * p.HW * p.heads;
  const long long cap = (long long)sm_count();       // one persistent CTA per SM
  const unsigned grid = (unsigned)(units < cap ? units : cap);
  attn_time_short_kernel<D, TB><<<grid, C::THREADS, C::SMEM_BYTES, stream>>>(mq, mk, mv, p);
  return last_launch_status();
}

template <int D>
int dispatch_time_short(const void* q, const void* k, const void* v, const TimeParams& p,
                           cudaStream_t stream) {
  // box rows: T rounded up to 8 (16 at least), from the set compiled here
  if (p.T <= 16) return launch_time_short<D, 16>(q, k, v, p, stream);
  if (p.T <= 24) return launch_time_short<D, 24>(q, k, v, p, stream);
  if (p.T <= 32) return launch_time_short<D, 32>(q, k, v, p, stream);
  if (p.T <= 48) return launch_time_short<D, 48>(q, k, v, p, stream);
  return launch_time_short<D, 64>(q, k, v, p, stream);
}

float resolve_scale(float scale, int D) { return scale > 0.f ? scale : 1.0f / std::sqrt((float)D); }

// Self-check of the bounded wait: one thread waits on an mbarrier that nothing
// will ever arrive on, so the wait runs out after kWaitLimitNs (or at once if
// the flag is already set) and records `site`, exactly as a stalled pipeline
// inside one of the library's kernels would.  Nothing faults and nothing is
// left in flight; the host reads the flag with vdit_device_status.
__global__ void watchdog_selftest_kernel(int site) {
  __shared__ uint64_t bar;
  if (threadIdx.x != 0) return;
  mbar_init(&bar, 1);
  fence_mbar_init();
  mbar_wait(&bar, 0, site);
}

int check_attn_args(const void* q, const void* k, const void* v, const void* o, const float* lse, long long B,
                    long long L, int heads, int D) {
  if (!q || !k || !v || !o) return VDIT_ERR_NULL;
  if (B <= 0 || L <= 0 || heads <= 0 || D <= 0) return VDIT_ERR_SHAPE;
  if (D != 32 && D != 64 && D != 128) return VDIT_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return VDIT_ERR_ALIGN;
  if (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u) != 0) return VDIT_ERR_ALIGN;
  // element offsets stay below 2^62 and tensor-map extents below 2^32
  if ((double)B * (double)L * (double)heads * (double)D > 4.0e18 || L > 0xffffffffLL || B > 0xffffffffLL)
    return VDIT_ERR_SHAPE;
  return VDIT_OK;
}

}  // namespace

extern "C" {

int vdit_version(void) { return 10100; }

const char* vdit_status_string(int status) {
  switch (status) {
    case VDIT_OK: return "ok";
    case VDIT_ERR_NULL: return "a required pointer is NULL";
    case VDIT_ERR_SHAPE: return "a size is non-positive, inconsistent or too large";
    case VDIT_ERR_ALIGN: return "a pointer is not 16-byte aligned";
    case VDIT_ERR_UNSUPPORTED: return "valid input this build does not handle";
    case VDIT_ERR_CUDA: return "the CUDA runtime reported an error";
    case VDIT_ERR_TIMEOUT: return "a bounded wait inside a kernel ran out";
    default: return "unknown status";
  }
}

int vdit_watchdog_selftest(int site, vdit_stream_t stream) {
  if (site < 1 || site > 255) return VDIT_ERR_SHAPE;
  watchdog_selftest_kernel<<<1, 32, 0, stream>>>(site);
  return last_launch_status();
}

int vdit_device_status(unsigned int* flags) {
  if (cudaDeviceSynchronize() != cudaSuccess) return VDIT_ERR_CUDA;
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_watchdog, sizeof(v)) != cudaSuccess) return VDIT_ERR_CUDA;
  if (flags != nullptr) *flags = v;
  if (v != 0) {
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbol(g_watchdog, &zero, sizeof(zero)) != cudaSuccess) return VDIT_ERR_CUDA;
    return VDIT_ERR_TIMEOUT;
  }
  return VDIT_OK;
}

int vdit_patchify_3d(const void* latent, void* tokens, int dtype, int N, int C, int T, int H, int W, int pt, int ph,
                     int pw, vdit_stream_t stream) {
  if (!latent || !tokens) return VDIT_ERR_NULL;
  if (dtype != VDIT_F32 && dtype != VDIT_BF16) return VDIT_ERR_UNSUPPORTED;
  if (N <= 0 || C <= 0 || T <= 0 || H <= 0 || W <= 0 || pt <= 0 || ph <= 0 || pw <= 0) return VDIT_ERR_SHAPE;
  PatchifyShape s;
  s.N = N; s.C = C; s.T = T; s.H = H; s.W = W; s.pt = pt; s.ph = ph; s.pw = pw;
  s.Tg = T / pt; s.Hg = H / ph; s.Wg = W / pw;
  if (s.Tg == 0 || s.Hg == 0 || s.Wg == 0) return VDIT_ERR_SHAPE;
  const long long F = (long long)C * pt * ph * pw;
  const long long ntok = (long long)N * s.Tg * s.Hg * s.Wg;
  if (ntok > 0x7fffffffLL || F > 0x7fffffffLL || (double)ntok * (double)F > 4.0e18) return VDIT_ERR_SHAPE;
  const int esz = dtype == VDIT_F32 ? 4 : 2;
  const long long brick_bytes = F * esz;
  constexpr long long kStage = 32 * 1024;          // staged latent rows per CTA
  // shared memory: staged rows (<= 2 * kStage with the padding) + offset table (<= kStage)
  if (brick_bytes > kStage || F * 4 > kStage) return VDIT_ERR_UNSUPPORTED;
  s.F = (int)F;
  s.WC = (int)std::min<long long>(s.Wg, kStage / brick_bytes);
  s.n_wchunks = (s.Wg + s.WC - 1) / s.WC;
  const long long rowlen = (long long)s.WC * pw + ((s.WC * pw) % 2 == 0 ? 1 : 0);   // odd staged row stride
  const int smem = (int)(((F * 4 + 15) & ~15LL) + (long long)C * pt * ph * rowlen * esz);
  const long long jobs = (long long)N * s.Tg * s.Hg * s.n_wchunks;
  const long long cap = (long long)sm_count() * 16;
  const unsigned grid = (unsigned)(jobs < cap ? jobs : cap);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  {
    // staged rows (<= 32 KB plus one element per row) plus the feature offset table (<= 32 KB)
    static bool done_f[kMaxDevices] = {}, done_b[kMaxDevices] = {};
    static std::mutex mu;
    std::lock_guard<std::mutex> lock(mu);
    if (!ensure_smem(patchify3d_kernel<float>, 3 * kStage + 16, done_f) ||
        !ensure_smem(patchify3d_kernel<__nv_bfloat16>, 3 * kStage + 16, done_b))
      return VDIT_ERR_CUDA;
  }
  // (every staged row must start 16-byte aligned: W a multiple of 4, and each chunk's
  // first column 2*w0 too, which holds with one chunk or an even chunk width)
  if (dtype == VDIT_F32 && pt == 1 && ph == 2 && pw == 2 && W % 4 == 0 && (s.n_wchunks == 1 || s.WC % 2 == 0) &&
      aligned16(latent) && aligned16(tokens)) {
    // the (1, 2, 2) float32 fast path: 2*C staged rows of 2*WC + 2 floats
    const int smem122 = (int)(2LL * C * (2LL * s.WC + 2) * 4);
    const long long cap122 = (long long)sm_count() * kPatchify122CtasPerSm;
    const unsigned grid122 = (unsigned)(jobs < cap122 ? jobs : cap122);
    if (smem122 > 48 * 1024) {
      static bool done[kMaxDevices] = {};
      static std::mutex mu2;
      std::lock_guard<std::mutex> lock(mu2);
      if (!ensure_smem(patchify122_f32_kernel, 3 * kStage + 16, done)) return VDIT_ERR_CUDA;
    }
    patchify122_f32_kernel<<<grid122, kPatchify122Threads, smem122, st>>>(static_cast<const float*>(latent),
                                                                      static_cast<float*>(tokens), s);
  } else if (dtype == VDIT_F32)
    patchify3d_kernel<float><<<grid, kPatchifyThreads, smem, st>>>(static_cast<const float*>(latent),
                                                                   static_cast<float*>(tokens), s);
  else
    patchify3d_kernel<__nv_bfloat16><<<grid, kPatchifyThreads, smem, st>>>(
        static_cast<const __nv_bfloat16*>(latent), static_cast<__nv_bfloat16*>(tokens), s);
  return last_launch_status();
}

int vdit_unpatchify_3d(const void* tokens, void* latent, int dtype, int N, int C, int Tg, int Hg, int Wg, int pt,
                       int ph, int pw, vdit_stream_t stream) {
  if (!tokens || !latent) return VDIT_ERR_NULL;
  if (dtype != VDIT_F32 && dtype != VDIT_BF16) return VDIT_ERR_UNSUPPORTED;
  if (N <= 0 || C <= 0 || Tg <= 0 || Hg <= 0 || Wg <= 0 || pt <= 0 || ph <= 0 || pw <= 0) return VDIT_ERR_SHAPE;
  const long long F = (long long)C * pt * ph * pw;
  const long long ntok = (long long)N * Tg * Hg * Wg;
  if (ntok > 0x7fffffffLL || F > 0x7fffffffLL || (double)ntok * (double)F > 4.0e18 ||
      (long long)Tg * pt > 0x7fffffffLL || (long long)Hg * ph > 0x7fffffffLL || (long long)Wg * pw > 0x7fffffffLL)
    return VDIT_ERR_SHAPE;
  const int esz = dtype == VDIT_F32 ? 4 : 2;
  constexpr long long kStage = 32 * 1024;
  if ((F + 1) * esz > kStage) return VDIT_ERR_UNSUPPORTED;
  UnpatchifyShape s;
  s.N = N; s.C = C; s.pt = pt; s.ph = ph; s.pw = pw; s.Tg = Tg; s.Hg = Hg; s.Wg = Wg; s.F = (int)F;
  s.WC = (int)std::min<long long>(Wg, kStage / ((F + 1) * esz));
  s.n_wchunks = (Wg + s.WC - 1) / s.WC;
  const int smem = (int)((long long)s.WC * (F + 1) * esz);
  const long long jobs = (long long)N * Tg * Hg * s.n_wchunks;
  const long long cap = (long long)sm_count() * 8;
  const unsigned grid = (unsigned)(jobs < cap ? jobs : cap);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // 16-byte loads when every token starts 16-byte aligned; paired stores when
  // pw == 2 and every brick's pair is aligned (W = Wg * 2 is even)
  const bool vec_in = aligned16(tokens) && (F * esz) % 16 == 0;
  const bool pair_out = pw == 2 && (reinterpret_cast<uintptr_t>(latent) % (2 * esz)) == 0;
  if (dtype == VDIT_F32)
    unpatchify3d_kernel<float><<<grid, kUnpatchifyThreads, smem, st>>>(static_cast<const float*>(tokens),
                                                                      static_cast<float*>(latent), s, vec_in,
                                                                      pair_out);
  else
    unpatchify3d_kernel<__nv_bfloat16><<<grid, kUnpatchifyThreads, smem, st>>>(
        static_cast<const __nv_bfloat16*>(tokens), static_cast<__nv_bfloat16*>(latent), s, vec_in, pair_out);
  return last_launch_status();
}

int vdit_patch_embed_3d(const float* latent, const void* weight, const float* bias, void* out, int N, int C, int T,
                        int H, int W, int pt, int ph, int pw, int dim, vdit_stream_t stream) {
  if (!latent || !weight || !out) return VDIT_ERR_NULL;
  if (N <= 0 || C <= 0 || T <= 0 || H <= 0 || W <= 0 || pt <= 0 || ph <= 0 || pw <= 0 || dim <= 0)
    return VDIT_ERR_SHAPE;
  const int Tg = T / pt, Hg = H / ph, Wg = W / pw;
  if (Tg == 0 || Hg == 0 || Wg == 0) return VDIT_ERR_SHAPE;
  if ((long long)C * pt * ph * pw != kEmbK || dim % kEmbBN != 0) return VDIT_ERR_UNSUPPORTED;
  if (!aligned16(weight) || !aligned16(out) || (bias && !aligned16(bias)) ||
      (reinterpret_cast<uintptr_t>(latent) & 3u) != 0)
    return VDIT_ERR_ALIGN;
  const long long ntok = (long long)N * Tg * Hg * Wg;
  if ((double)N * C * T * (double)H * W > 4.0e18 || (double)ntok * dim > 4.0e18 ||
      (ntok + kEmbBM - 1) / kEmbBM > 0x7fffffffLL)
    return VDIT_ERR_SHAPE;
  static bool smem_done[kMaxDevices] = {};
  static std::mutex mu;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (!ensure_smem(patch_embed_kernel, kEmbSmem, smem_done)) return VDIT_ERR_CUDA;
  }
  CUtensorMap mw, mo;
  if (!make_2d_map(&mw, weight, kEmbK, dim, kEmbK, kEmbBN) || !make_2d_map(&mo, out, dim, ntok, kEmbOutBox, 32))
    return VDIT_ERR_CUDA;
  EmbedParams p;
  p.latent = latent; p.bias = bias; p.out = static_cast<__nv_bfloat16*>(out);
  p.C = C; p.T = T; p.H = H; p.W = W; p.pt = pt; p.ph = ph; p.pw = pw; p.Tg = Tg; p.Hg = Hg; p.Wg = Wg;
  p.ntok = ntok; p.dim = dim;
  p.n_mt = (int)((ntok + kEmbBM - 1) / kEmbBM);
  const int n_nt = dim / kEmbBN;
  p.group_nt = (n_nt + 3) / 4;                         // up to four work items per token tile
  p.n_groups = (n_nt + p.group_nt - 1) / p.group_nt;
  if ((long long)p.n_mt * p.n_groups > 0x7fffffffLL) return VDIT_ERR_SHAPE;
  p.n_items = p.n_mt * p.n_groups;
  const long long sms = sm_count();
  const unsigned grid = (unsigned)(p.n_items < sms ? p.n_items : sms);
  patch_embed_kernel<<<grid, kEmbThreads, kEmbSmem, reinterpret_cast<cudaStream_t>(stream)>>>(mw, mo, p);
  return last_launch_status();
}

int vdit_rope_3d(const void* q_in, const void* k_in, void* q_out, void* k_out, int B, int Tg, int Hg, int Wg,
                 int heads, int head_dim, int d_t, int d_h, int d_w, float theta, vdit_stream_t stream) {
  const bool k_only = q_in == nullptr && q_out == nullptr;
  if (k_only) { q_in = k_in; q_out = k_out; }
  if (!q_in || !k_in || !q_out || !k_out) return VDIT_ERR_NULL;
  if (B <= 0 || Tg <= 0 || Hg <= 0 || Wg <= 0 || heads <= 0 || head_dim <= 0) return VDIT_ERR_SHAPE;
  if (d_t < 0 || d_h < 0 || d_w < 0 || (d_t | d_h | d_w) & 1 || d_t + d_h + d_w != head_dim) return VDIT_ERR_SHAPE;
  if (!(theta > 0.f) || !std::isfinite(theta)) return VDIT_ERR_SHAPE;
  if (head_dim % 8 != 0 || head_dim / 2 > kRopeMaxPairs) return VDIT_ERR_UNSUPPORTED;
  if (!aligned16(q_in) || !aligned16(k_in) || !aligned16(q_out) || !aligned16(k_out)) return VDIT_ERR_ALIGN;
  const long long L = (long long)Tg * Hg * Wg;
  if (L > 0x7fffffffLL || (double)B * (double)L * heads * head_dim > 4.0e18) return VDIT_ERR_SHAPE;
  RopeShape s;
  s.ntok = (long long)B * L;
  s.L = (int)L; s.Hg = Hg; s.Wg = Wg;
  s.heads = heads; s.D = head_dim;
  s.pt_end = d_t / 2; s.ph_end = (d_t + d_h) / 2;
  s.d_t = d_t; s.d_h = d_h; s.d_w = d_w;
  s.ntens = k_only ? 1 : 2;
  const long long want = (s.ntok + kRopeTokens - 1) / kRopeTokens;
  const long long cap = (long long)sm_count() * 8;
  const unsigned grid = (unsigned)(want < cap ? want : cap);
  rope3d_kernel<<<grid, kRopeThreads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<const __nv_bfloat16*>(q_in), static_cast<const __nv_bfloat16*>(k_in),
      static_cast<__nv_bfloat16*>(q_out), static_cast<__nv_bfloat16*>(k_out), s, (double)theta);
  return last_launch_status();
}

int vdit_qk_norm_rope_3d(const void* q_in, const void* k_in, void* q_out, void* k_out, const float* wq,
                         const float* wk, int norm_group, float eps, int B, int Tg, int Hg, int Wg, int heads,
                         int head_dim, int d_t, int d_h, int d_w, float theta, vdit_stream_t stream) {
  const bool k_only = q_in == nullptr && q_out == nullptr;
  if (k_only) { q_in = k_in; q_out = k_out; }
  if (!q_in || !k_in || !q_out || !k_out) return VDIT_ERR_NULL;
  if (B <= 0 || Tg <= 0 || Hg <= 0 || Wg <= 0 || heads <= 0 || head_dim <= 0) return VDIT_ERR_SHAPE;
  if (d_t < 0 || d_h < 0 || d_w < 0 || (d_t | d_h | d_w) & 1 || d_t + d_h + d_w != head_dim) return VDIT_ERR_SHAPE;
  if (!(theta > 0.f) || !std::isfinite(theta)) return VDIT_ERR_SHAPE;
  const long long width = (long long)heads * head_dim;
  if (norm_group <= 0 || width % norm_group != 0 || !(eps >= 0.f) || !std::isfinite(eps)) return VDIT_ERR_SHAPE;
  if (head_dim % 8 != 0 || head_dim / 2 > kRopeMaxPairs || norm_group % 8 != 0) return VDIT_ERR_UNSUPPORTED;
  const int gv = norm_group / 8;                       // 16-byte vectors per group
  const bool wide = norm_group == width;               // one group: the token's whole vector
  if (!wide && 32 % gv != 0) return VDIT_ERR_UNSUPPORTED;
  if (width > 128LL * 8 * kNormVecs) return VDIT_ERR_UNSUPPORTED;
  if (!aligned16(q_in) || !aligned16(k_in) || !aligned16(q_out) || !aligned16(k_out) ||
      (wq && !aligned16(wq)) || (wk && !aligned16(wk)))
    return VDIT_ERR_ALIGN;
  const long long L = (long long)Tg * Hg * Wg;
  if (L > 0x7fffffffLL || (double)B * (double)L * (double)width > 4.0e18) return VDIT_ERR_SHAPE;
  RopeShape s;
  s.ntok = (long long)B * L;
  s.L = (int)L; s.Hg = Hg; s.Wg = Wg;
  s.heads = heads; s.D = head_dim;
  s.pt_end = d_t / 2; s.ph_end = (d_t + d_h) / 2;
  s.d_t = d_t; s.d_h = d_h; s.d_w = d_w;
  s.ntens = k_only ? 1 : 2;
  const long long cap = (long long)sm_count() * 2;
  const unsigned grid = (unsigned)(s.ntok < cap ? s.ntok : cap);
  // the ring (Q and K rows of kNormStages tokens) and the per-axis (cos, sin) tables
  const long long tab = (long long)Tg * (d_t / 2) + (long long)Hg * (d_h / 2) + (long long)Wg * (d_w / 2);
  if (tab > kNormMaxTable) return VDIT_ERR_UNSUPPORTED;
  const int smem = kNormStages * 2 * (int)width * 2 + (int)tab * 8;
  {
    static bool done_n[kMaxDevices] = {}, done_w[kMaxDevices] = {};
    static std::mutex mu;
    std::lock_guard<std::mutex> lock(mu);
    if (!ensure_smem(qk_norm_rope3d_kernel<false>, kNormStages * 2 * 8192 * 2 + kNormMaxTable * 8, done_n) ||
        !ensure_smem(qk_norm_rope3d_kernel<true>, kNormStages * 2 * 8192 * 2 + kNormMaxTable * 8, done_w))
      return VDIT_ERR_CUDA;
  }
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const auto* qi = static_cast<const __nv_bfloat16*>(q_in);
  const auto* ki = static_cast<const __nv_bfloat16*>(k_in);
  auto* qo = static_cast<__nv_bfloat16*>(q_out);
  auto* ko = static_cast<__nv_bfloat16*>(k_out);
  if (wide)
    qk_norm_rope3d_kernel<true><<<grid, kNormThreads, smem, st>>>(qi, ki, qo, ko, wq, wk, s, norm_group, eps,
                                                               (double)theta);
  else
    qk_norm_rope3d_kernel<false><<<grid, kNormThreads, smem, st>>>(qi, ki, qo, ko, wq, wk, s, norm_group, eps,
                                                                (double)theta);
  return last_launch_status();
}

int vdit_attn_full(const void* q, const void* k, const void* v, void* o, float* lse, int B, int L, int heads,
                   int head_dim, float scale, vdit_stream_t stream) {
  const int rc = check_attn_args(q, k, v, o, lse, B, L, heads, head_dim);
  if (rc != VDIT_OK) return rc;
  return dispatch_tcgen05(head_dim, q, k, v, o, lse, kSeq, B, L, L, 1, heads, resolve_scale(scale, head_dim),
                          reinterpret_cast<cudaStream_t>(stream));
}

long long vdit_rope_3d_table_entries(int Tg, int Hg, int Wg, int head_dim, int d_t, int d_h, int d_w) {
  if (check_rope_shape(Tg, Hg, Wg, head_dim, d_t, d_h, d_w, 1.f) != VDIT_OK) return -1;
  return rope_table_entries(Tg, Hg, Wg, d_t, d_h, d_w);
}

int vdit_rope_3d_table(float* table, int Tg, int Hg, int Wg, int head_dim, int d_t, int d_h, int d_w, float theta,
                       vdit_stream_t stream) {
  if (!table) return VDIT_ERR_NULL;
  const int rc = check_rope_shape(Tg, Hg, Wg, head_dim, d_t, d_h, d_w, theta);
  if (rc != VDIT_OK) return rc;
  if (!aligned16(table)) return VDIT_ERR_ALIGN;
  const long long n = rope_table_entries(Tg, Hg, Wg, d_t, d_h, d_w);
  if (n > 0x7fffffffLL) return VDIT_ERR_SHAPE;
  if (n == 0) return VDIT_OK;
  const long long blocks = (n + 255) / 256;
  const long long cap = (long long)sm_count() * 4;
  rope3d_table_kernel<<<(unsigned)(blocks < cap ? blocks : cap), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      reinterpret_cast<float2*>(table), Tg, Hg, Wg, d_t, d_h, d_w, (double)theta);
  return last_launch_status();
}

int vdit_attn_full_rope_q(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Tg, int Hg,
                          int Wg, int heads, int head_dim, float scale, int d_t, int d_h, int d_w,
                          const float* rope_table, const float* wq, int norm_group, float eps,
                          vdit_stream_t stream) {
  if (!rope_table) return VDIT_ERR_NULL;
  if (Tg <= 0 || Hg <= 0 || Wg <= 0) return (!q || !k || !v || !o) ? VDIT_ERR_NULL : VDIT_ERR_SHAPE;
  const long long L = (long long)Tg * Hg * Wg;
  int rc = check_attn_args(q, k, v, o, lse, B, L, heads, head_dim);
  if (rc != VDIT_OK) return rc;
  rc = check_rope_shape(Tg, Hg, Wg, head_dim, d_t, d_h, d_w, 1.f);
  if (rc != VDIT_OK) return rc;
  if (norm_group != 0 && norm_group != head_dim) return VDIT_ERR_UNSUPPORTED;
  if (norm_group != 0 && (!(eps >= 0.f) || !std::isfinite(eps))) return VDIT_ERR_SHAPE;
  if (!aligned16(rope_table) || (wq && !aligned16(wq))) return VDIT_ERR_ALIGN;
  // the kernel stages the table, then the norm's head_dim weights, in one K/V
  // ring stage: 128 x head_dim bf16
  if (rope_table_entries(Tg, Hg, Wg, d_t, d_h, d_w) * 8 + head_dim * 4 > 128LL * head_dim * 2)
    return VDIT_ERR_UNSUPPORTED;
  AttnParams r{};
  r.rope_tab = reinterpret_cast<const float2*>(rope_table);
  r.wq = wq;
  r.rope_tg = Tg; r.rope_hg = Hg; r.rope_wg = Wg;
  r.rope_pt = d_t / 2; r.rope_ph = d_h / 2;
  r.rope_off_h = Tg * (d_t / 2);
  r.rope_off_w = r.rope_off_h + Hg * (d_h / 2);
  r.rope_n = (int)rope_table_entries(Tg, Hg, Wg, d_t, d_h, d_w);
  r.norm = norm_group != 0;
  r.eps = eps;
  r.inv_d = 1.f / (float)head_dim;
  return dispatch_tcgen05(head_dim, q, k, v, o, lse, kSeq, B, (int)L, (int)L, 1, heads,
                          resolve_scale(scale, head_dim), reinterpret_cast<cudaStream_t>(stream), &r);
}

int vdit_attn_cross(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Lq, int Lk,
                    int heads, int head_dim, float scale, vdit_stream_t stream) {
  int rc = check_attn_args(q, k, v, o, lse, B, Lq, heads, head_dim);
  if (rc == VDIT_OK) rc = check_attn_args(q, k, v, o, lse, B, Lk, heads, head_dim);
  if (rc != VDIT_OK) return rc;
  return dispatch_tcgen05(head_dim, q, k, v, o, lse, kSeq, B, Lq, Lk, 1, heads, resolve_scale(scale, head_dim),
                          reinterpret_cast<cudaStream_t>(stream));
}

int vdit_attn_divided_space(const void* q, const void* k, const void* v, void* o, float* lse, int B, int T, int HW,
                            int heads, int head_dim, float scale, vdit_stream_t stream) {
  if (T <= 0 || HW <= 0 || B <= 0) return (!q || !k || !v || !o) ? VDIT_ERR_NULL : VDIT_ERR_SHAPE;
  const int rc = check_attn_args(q, k, v, o, lse, (long long)B * T, HW, heads, head_dim);
  if (rc != VDIT_OK) return rc;
  if ((long long)B * T > 0x7fffffffLL) return VDIT_ERR_SHAPE;
  return dispatch_tcgen05(head_dim, q, k, v, o, lse, kSeq, B * T, HW, HW, T, heads, resolve_scale(scale, head_dim),
                          reinterpret_cast<cudaStream_t>(stream));
}

int vdit_attn_divided_time(const void* q, const void* k, const void* v, void* o, float* lse, int B, int T, int HW,
                           int heads, int head_dim, float scale, vdit_stream_t stream) {
  if (T <= 0 || HW <= 0 || B <= 0) return (!q || !k || !v || !o) ? VDIT_ERR_NULL : VDIT_ERR_SHAPE;
  const int rc = check_attn_args(q, k, v, o, lse, (long long)B * HW, T, heads, head_dim);
  if (rc != VDIT_OK) return rc;
  if ((long long)B * HW > 0x7fffffffLL || (long long)T * HW > 0x7fffffffLL) return VDIT_ERR_SHAPE;
  const float sc = resolve_scale(scale, head_dim);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (T > 64)  // long clips: the tensor-core kernel over a strided view, one sequence per site
    return dispatch_tcgen05(head_dim, q, k, v, o, lse, kTime, B * HW, T, T, HW, heads, sc, st);
  TimeParams p;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.B = B; p.T = T; p.HW = HW; p.heads = heads;
  p.scale_log2 = sc * 1.4426950408889634f;
  switch (head_dim) {
    case 32: return dispatch_time_short<32>(q, k, v, p, st);
    case 64: return dispatch_time_short<64>(q, k, v, p, st);
    case 128: return dispatch_time_short<128>(q, k, v, p, st);
    default: return VDIT_ERR_UNSUPPORTED;
  }
}

}  // extern "C"
