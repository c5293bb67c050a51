// Host side of the C ABI (include/xlpk.h): validation, the ahead-of-time
// planner (static partition of every stage over the CTAs, weight packing in
// stream order, RoPE table, workspace), and the launches.
//
// The planner is the "AOT" half of the design the pages describe: the model is
// unrolled ahead of time into a fixed schedule of tile tasks whose shapes,
// placement and residency are decided before the first token ("Ultra-High
// Interactivity On NVIDIA GPUs? - TileRT InferenceX", digest, core views: the
// decode graph is statically compiled into one resident Engine Kernel; the
// fixed temporary-tensor table of "Persistent execution paradigm", section
// 5.3, becomes the static workspace arena below).
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <chrono>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/xlpk.h"
#include "engine.cuh"
#include "kernels.h"
#include "params.h"

using namespace xlpk;

namespace {

thread_local std::string g_cuda_err;

xlpk_status cuda_fail(cudaError_t e, const char* what) {
  g_cuda_err = std::string(what) + ": " + cudaGetErrorString(e);
  return e == cudaErrorMemoryAllocation ? XLPK_ERR_OOM : XLPK_ERR_CUDA;
}

#define XLPK_CUDA(call)                               \
  do {                                                \
    cudaError_t e_ = (call);                          \
    if (e_ != cudaSuccess) return cuda_fail(e_, #call); \
  } while (0)

struct PackJob {
  const uint8_t* src;   // source row
  const void* scale;    // FP8: the row's block-scale row ([K/128] fp32); NVFP4: [K/16] e4m3; else null
  long long base;       // byte offset of the CTA's span in the packed buffer
  int row;              // row inside its tile (2 * pair-in-group + 0/1)
  int j16;              // rows of the span before this row's group
  int gp2;              // rows of this row's group
  int np2;              // rows of the span
};

// Where chunk kc of a packed row starts.  The span's tiles are ordered
// (window, group, chunk in window); with one window (cw = nkc) this is the
// plain (group, chunk) order.  Returns the tile's offset; the row's codes sit
// at + row * KC * esz, an FP8 tile's scales at + gp2 * KC + row * KC / 32.
__host__ __device__ inline long long pack_tile_offset(const PackJob& j, int kc, int nkc, int cw, long long tile_row) {
  const int w = kc / cw;
  const int cww = (nkc - w * cw) < cw ? (nkc - w * cw) : cw;
  return j.base + static_cast<long long>(j.np2) * cw * w * tile_row + static_cast<long long>(j.j16) * cww * tile_row +
         static_cast<long long>(kc - w * cw) * j.gp2 * tile_row;
}

// bf16 [R][C] row-major -> [C][R] row-major (32x32 tiles through shared memory).
__global__ void transpose_bf16_kernel(const uint16_t* in, uint16_t* out, int R, int C) {
  __shared__ uint16_t t[32][33];
  const int c0 = blockIdx.x * 32, r0 = blockIdx.y * 32;
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int r = r0 + i, c = c0 + threadIdx.x;
    if (r < R && c < C) t[i][threadIdx.x] = in[static_cast<size_t>(r) * C + c];
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int c = c0 + i, r = r0 + threadIdx.x;
    if (r < R && c < C) out[static_cast<size_t>(c) * R + r] = t[threadIdx.x][i];
  }
}

// FP8: one thread per (row, chunk): the chunk's KC/128 block scales of the row.
__global__ void pack_scales_kernel(const PackJob* jobs, int njobs, uint8_t* out, int nchunk, int kc_cols, int cw,
                                   long long tile_row) {
  const long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= static_cast<long long>(njobs) * nchunk) return;
  const int jb = static_cast<int>(t / nchunk), c = static_cast<int>(t - static_cast<long long>(jb) * nchunk);
  const PackJob j = jobs[jb];
  const int kb_per_chunk = kc_cols / 128;
  float* d = reinterpret_cast<float*>(out + pack_tile_offset(j, c, nchunk, cw, tile_row) +
                                      static_cast<long long>(j.gp2) * kc_cols + j.row * (kc_cols / 32));
  const float* sr = static_cast<const float*>(j.scale);
  for (int k = 0; k < kb_per_chunk; ++k) d[k] = sr[c * kb_per_chunk + k];
}

// NVFP4: one thread per (row, chunk): the chunk's KC/16 e4m3 block scales of
// the row, after the tile's code rows ([gp2 rows][KC/2 bytes]).
__global__ void pack_scales4_kernel(const PackJob* jobs, int njobs, uint8_t* out, int nchunk, int kc_cols, int cw,
                                    long long tile_row) {
  const long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= static_cast<long long>(njobs) * nchunk) return;
  const int jb = static_cast<int>(t / nchunk), c = static_cast<int>(t - static_cast<long long>(jb) * nchunk);
  const PackJob j = jobs[jb];
  const int nb = kc_cols / 16;
  uint8_t* d = out + pack_tile_offset(j, c, nchunk, cw, tile_row) + static_cast<long long>(j.gp2) * (kc_cols / 2) +
               static_cast<long long>(j.row) * nb;
  const uint8_t* sr = static_cast<const uint8_t*>(j.scale) + static_cast<long long>(c) * nb;
  for (int k = 0; k < nb; ++k) d[k] = sr[k];
}

// One warp per packed row: chunk c of the row goes to its tile (pack_tile_offset).
__global__ void pack_rows_kernel(const PackJob* jobs, int njobs, uint8_t* out, int row_bytes, int chunk_bytes,
                                 int nchunk, int cw, long long tile_row) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= njobs) return;
  const PackJob j = jobs[warp];
  const int nvec = row_bytes >> 4, nvc = chunk_bytes >> 4;
  const uint4* src = reinterpret_cast<const uint4*>(j.src);
  for (int v = lane; v < nvec; v += 32) {
    const int c = v / nvc, w = v - c * nvc;
    *reinterpret_cast<uint4*>(out + pack_tile_offset(j, c, nchunk, cw, tile_row) +
                              static_cast<long long>(j.row) * chunk_bytes + static_cast<long long>(w) * 16) = src[v];
  }
}

long long split_host(long long c, long long n, long long G) { return (c * n) / G; }

// ---- batch-8 tensor-core packing (params.h: "batch-8 tensor-core tiles")
struct TcRowJob {
  const uint8_t* src;   // source row (K codes or bf16 values)
  const float* scale;   // FP8: the row's block-scale row ([K/128] fp32), else null
  int n;                // logical row
};

static_assert(sizeof(TcRowJob) <= sizeof(PackJob), "the tensor-core packer reuses the job buffer");

struct TcGeom {
  int N, K, G, win, fp8;
};

// Byte offset of the tile holding column k of logical row n, and the row's
// M-tile geometry (rows rv, boxes per tile nb, box j, row r, column in window kw).
__device__ inline long long tc_tile_of(const TcGeom& g, int n, int k, int& rv, int& nb, int& j, int& r, int& kw) {
  const int U = g.N / 8;
  const int c = static_cast<int>(((static_cast<long long>(n / 8) + 1) * g.G - 1) / U);
  const int u0 = static_cast<int>((static_cast<long long>(c) * U) / g.G);
  const int u1 = static_cast<int>((static_cast<long long>(c + 1) * U) / g.G);
  const int R = 8 * (u1 - u0);
  const int lr = n - 8 * u0, m = lr / 128;
  r = lr % 128;
  rv = min(128, R - 128 * m);
  const int bc = tc_box_cols(g.fp8);
  nb = tc_nb(rv, tc_kbox(g.K, g.win, g.fp8), g.fp8);
  const int w = g.win > 0 ? k / g.win : 0;
  const int ws = w * g.win;
  const int Kw = g.win > 0 ? min(g.win, g.K - ws) : g.K;
  kw = k - ws;
  const int bw = kw / bc;
  j = bw % nb;
  return 8LL * u0 * tc_row_bytes(g.K, g.fp8) + static_cast<long long>(w) * R * tc_row_bytes(g.win, g.fp8) +
         128LL * m * tc_row_bytes(Kw, g.fp8) + static_cast<long long>(bw / nb) * tc_tile_bytes(rv, nb, g.fp8);
}

// One warp per row: its 16-byte units to their swizzled places.
__global__ void pack_tc_rows_kernel(const TcRowJob* jobs, int njobs, uint8_t* out, TcGeom g) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= njobs) return;
  const TcRowJob jb = jobs[warp];
  const int esz = g.fp8 ? 1 : 2;
  const int nvec = g.K * esz / 16, bc = tc_box_cols(g.fp8);
  const uint4* src = reinterpret_cast<const uint4*>(jb.src);
  for (int v = lane; v < nvec; v += 32) {
    const int k = v * 16 / esz;
    int rv, nb, j, r, kw;
    const long long t = tc_tile_of(g, jb.n, k, rv, nb, j, r, kw);
    const int q = ((kw % bc) * esz) / 16;
    *reinterpret_cast<uint4*>(out + t + static_cast<long long>(j) * rv * 128 + r * 128 + ((q ^ (r & 7)) << 4)) =
        src[v];
  }
}

// FP8: one thread per (row, 128-column block): the block scale after the tile's boxes.
__global__ void pack_tc_scales_kernel(const TcRowJob* jobs, int njobs, uint8_t* out, TcGeom g) {
  const long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int nkb = g.K / 128;
  if (t >= static_cast<long long>(njobs) * nkb) return;
  const int i = static_cast<int>(t / nkb), kb = static_cast<int>(t - static_cast<long long>(i) * nkb);
  const TcRowJob jb = jobs[i];
  int rv, nb, j, r, kw;
  const long long tile = tc_tile_of(g, jb.n, kb * 128, rv, nb, j, r, kw);
  *reinterpret_cast<float*>(out + tile + static_cast<long long>(nb) * rv * 128 + (static_cast<long long>(j) * rv + r) * 4) =
      jb.scale[kb];
}

// Largest k-chunk dividing K whose tile of 8 row pairs fits kTileBytes (FP8:
// also a whole number of 128-column scale blocks; NVFP4: rows of KC/2 code
// bytes + KC/16 scale bytes, KC a multiple of 128 so tiles stay 16-byte sized).
int pick_kc(int K, int esz, bool fp4 = false) {
  if (fp4) {
    for (int kc = std::min(K, kTileBytes * 16 / (2 * kPairsPerTile * 9)); kc >= 128; --kc)
      if (K % kc == 0 && kc % 128 == 0) return kc;
    return 0;
  }
  const int vec = esz == 1 ? 128 : 16 / esz;
  const int cap = kTileBytes / (2 * kPairsPerTile * esz);
  for (int kc = std::min(K, cap); kc >= vec; --kc)
    if (K % kc == 0 && kc % vec == 0) return kc;
  return 0;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

enum class MatKind { QKV, PLAIN, GATEUP };

struct MatSrc {
  MatKind kind;
  const uint8_t* a;   // QKV: wq; GATEUP: gate; PLAIN: w
  const uint8_t* b;   // QKV: wk; GATEUP: up
  const uint8_t* c;   // QKV: wv
  const void* sa = nullptr;   // block scales of a, b, c: FP8 fp32 [rows/128][K/128], NVFP4 e4m3 [rows][K/16]
  const void* sb = nullptr;
  const void* sc = nullptr;
  float ga = 1.f, gb = 1.f, gc = 1.f;   // NVFP4: the matrix scales of a, b, c
};

struct SrcRow {
  const uint8_t* w;
  const void* s;   // the row's block-scale row (FP8: fp32, NVFP4: e4m3), else null
  float g;         // NVFP4: the source matrix's scale
};

}  // namespace

struct xlpk_engine {
  xlpk_config cfg{};
  int device = 0;
  int G = 0;
  int nslot = 0;
  bool shallow = false;         // batch <= 4: kShallowSlots ring slots, kShallowPrefetchBytes of L2 prefetch
  int smem = 0;
  int act_bytes = 0;
  int side_bytes = 0, side_rope = 0, side_resid = 0, side_embed = 0, nvr = 0, rows_side = 0, evb = 0;
  int side_hloc = 0, hloc = 0;
  bool ffn_fused = false;
  bool tc = false;              // batch-8 projections on tcgen05 MMAs
  int tc_cols = 0;
  int down_win = 0;            // K-windowed down projection (columns per window; 0: off)
  int tc_win = 0;              // K window of the tensor-core projections (0: whole K)
  int esz = 2;                 // bytes per weight element (1: e4m3 codes, or NVFP4 with fp4 set)
  bool fp4 = false;            // NVFP4 weights
  int P = 0;
  uint8_t* packed = nullptr;
  size_t packed_bytes = 0;
  uint8_t* ws = nullptr;
  size_t ws_bytes = 0;
  LayerParams* d_layers = nullptr;
  float2* rope = nullptr;
  int32_t* tok_scratch = nullptr;
  Params base{};
  std::vector<int> pos;
  int step_base = 0;
  cudaStream_t last_stream = nullptr;
  const void* kern_persistent = nullptr;
  const void* kern_stage = nullptr;
  void (*launch_stage)(const Params&, int, int, int, int, int, cudaStream_t) = nullptr;
  int64_t weight_bytes_per_step = 0;
  float* dbg_logits = nullptr;   // parity mode (xlpk_debug_logits): [B][V], [B][H], last step's
  float* dbg_hidden = nullptr;
  // serve mode (xlpk_serve_*)
  unsigned* serve_ctl = nullptr;     // host-mapped words: [0] requested, [1] leave, [2] done
  int32_t* serve_tokens = nullptr;   // host-mapped token ring [serve_cap][B]
  unsigned* serve_ctl_dev = nullptr; // the same memory as the device sees it
  int32_t* serve_tokens_dev = nullptr;
  int serve_cap = 0;
  bool serve_active = false;         // a session is open
  bool serve_launched = false;       // a serve launch may still be running
  cudaStream_t serve_stream = nullptr;
  long long serve_posted = 0;        // steps requested in the session
  long long serve_step0 = 0;         // session steps done before the current launch
  long long serve_idle_ns = 0;
  unsigned* serve_dev_words = nullptr;   // workspace: [0] forwarded request count, [1] stop step
  int32_t* verify_word = nullptr;        // workspace: tokens emitted by the last verify step
};

namespace {

// Dense and MoE models use separate kernel instantiations, so the dense
// kernels carry none of the routing code; likewise bf16 and e4m3 caches, so
// the bf16 kernels carry none of the e4m3 code (nor its register pressure).
template <int B, int D, bool MOE = false, int VAR = 0>
void bind_kernels(xlpk_engine* e) {
  const KernelSet k = kernel_set<B, D, MOE, VAR>();
  e->kern_persistent = k.persistent;
  e->kern_stage = k.stage;
  e->launch_stage = k.launch_stage;
}

// var: bit 0 an e4m3 KV cache, bit 1 NVFP4 weights (batch 1, dense).
bool bind_by_shape(xlpk_engine* e, int B, int D, bool moe, int var) {
  if (moe) {   // MoE is built for batch 1 with bf16 / e4m3 weights and a bf16 cache
    if (var != 0) return false;
    if (B == 1 && D == 64) return bind_kernels<1, 64, true>(e), true;
    if (B == 1 && D == 128) return bind_kernels<1, 128, true>(e), true;
    return false;
  }
  if (var & 2) {
    if (B != 1) return false;
    if (D == 64) return (var & 1 ? bind_kernels<1, 64, false, 3>(e) : bind_kernels<1, 64, false, 2>(e)), true;
    if (D == 128) return (var & 1 ? bind_kernels<1, 128, false, 3>(e) : bind_kernels<1, 128, false, 2>(e)), true;
    return false;
  }
#define XLPK_BIND(b, d)                     \
  if (B == b && D == d) {                   \
    if (var & 1)                            \
      bind_kernels<b, d, false, 1>(e);      \
    else                                    \
      bind_kernels<b, d>(e);                \
    return true;                            \
  }
  XLPK_BIND(1, 64)
  XLPK_BIND(1, 128)
  XLPK_BIND(2, 64)
  XLPK_BIND(2, 128)
  XLPK_BIND(4, 64)
  XLPK_BIND(4, 128)
  XLPK_BIND(8, 64)
  XLPK_BIND(8, 128)
#undef XLPK_BIND
  return false;
}

// Logical row n of a packed matrix -> source row (and its block-scale row).
SrcRow source_row(const MatSrc& ms, long long n, int K, int esz, const xlpk_config& c, bool fp4 = false) {
  const long long row_bytes = fp4 ? K / 2 : static_cast<long long>(K) * esz;
  const long long pr = n >> 1;
  const int r = static_cast<int>(n & 1);
  const uint8_t* base = nullptr;
  const void* sbase = nullptr;
  float g = 1.f;
  long long row = 0;
  switch (ms.kind) {
    case MatKind::PLAIN:
      base = ms.a, sbase = ms.sa, g = ms.ga, row = n;
      break;
    case MatKind::GATEUP:
      base = r == 0 ? ms.a : ms.b, sbase = r == 0 ? ms.sa : ms.sb, g = r == 0 ? ms.ga : ms.gb, row = pr;
      break;
    case MatKind::QKV: {
      const long long half = c.head_dim / 2;
      const long long hq = static_cast<long long>(c.n_q_heads) * half;
      const long long hk = static_cast<long long>(c.n_kv_heads) * half;
      if (pr < hq + hk) {
        const bool isq = pr < hq;
        const long long pp = isq ? pr : pr - hq;
        const long long head = pp / half, i = pp % half;
        row = head * c.head_dim + i + r * half;
        base = isq ? ms.a : ms.b, sbase = isq ? ms.sa : ms.sb, g = isq ? ms.ga : ms.gb;
      } else {
        row = 2 * (pr - hq - hk) + r;
        base = ms.c, sbase = ms.sc, g = ms.gc;
      }
      break;
    }
  }
  SrcRow out;
  out.w = base + row * row_bytes;
  if (!sbase)
    out.s = nullptr;
  else if (fp4)
    out.s = static_cast<const uint8_t*>(sbase) + row * (K / 16);
  else
    out.s = static_cast<const float*>(sbase) + (row / 128) * (K / 128);
  out.g = g;
  return out;
}

// Pack one matrix into `dst` (device) in stream order; returns the Mat view.
// `split` CTAs share the rows (1: the whole matrix is one block streamed by
// every CTA that needs it, e.g. the MoE router and expert gate/up blocks).
xlpk_status pack_matrix(xlpk_engine* e, const MatSrc& ms, int N, int K, uint8_t* dst, Mat* out,
                        PackJob* d_jobs, size_t max_jobs, cudaStream_t st, int split, int win_cols = 0) {
  const int esz = e->esz;
  const bool fp4 = e->fp4 && esz == 1;   // (the MoE router stays bf16)
  const int KC = pick_kc(K, esz, fp4);
  if (KC == 0) return XLPK_ERR_UNSUPPORTED;
  const bool fp8 = esz == 1 && !fp4;
  if ((fp8 || fp4) && (!ms.sa || (ms.kind != MatKind::PLAIN && !ms.sb) || (ms.kind == MatKind::QKV && !ms.sc)))
    return XLPK_ERR_INVALID_ARG;
  const int nkc = K / KC;
  // chunks per window: the whole K unless the matrix is streamed window by window
  const int cw = win_cols > 0 ? win_cols / KC : nkc;
  if (cw < 1 || (win_cols > 0 && win_cols % KC)) return XLPK_ERR_UNSUPPORTED;
  // bytes per packed row over a chunk / over K (codes + block scales)
  const long long tile_row =
      fp4 ? KC / 2 + KC / 16 : static_cast<long long>(KC) * esz + (fp8 ? KC / 32 : 0);
  const long long full_row = fp4 ? K / 2 + K / 16 : static_cast<long long>(K) * esz + (fp8 ? K / 32 : 0);
  const long long NP = N / 2, G = split;
  std::vector<PackJob> jobs;
  jobs.reserve(static_cast<size_t>(N));
  for (long long c = 0; c < G; ++c) {
    const long long p0 = split_host(c, NP, G), p1 = split_host(c + 1, NP, G);
    const long long npc = p1 - p0;
    for (long long lp = 0; lp < npc; ++lp) {
      const long long j = lp / kPairsPerTile, w = lp % kPairsPerTile;
      const long long gp = std::min<long long>(kPairsPerTile, npc - kPairsPerTile * j);
      for (int r = 0; r < 2; ++r) {
        const SrcRow sr = source_row(ms, 2 * (p0 + lp) + r, K, esz, e->cfg, fp4);
        PackJob pj;
        pj.src = sr.w;
        pj.scale = sr.s;
        pj.base = 2 * p0 * full_row;
        pj.row = static_cast<int>(2 * w + r);
        pj.j16 = static_cast<int>(2 * kPairsPerTile * j);
        pj.gp2 = static_cast<int>(2 * gp);
        pj.np2 = static_cast<int>(2 * npc);
        jobs.push_back(pj);
      }
    }
  }
  const int row_bytes = fp4 ? K / 2 : K * esz, chunk_bytes = fp4 ? KC / 2 : KC * esz;
  for (size_t off = 0; off < jobs.size(); off += max_jobs) {
    const size_t n = std::min(max_jobs, jobs.size() - off);
    XLPK_CUDA(cudaMemcpyAsync(d_jobs, jobs.data() + off, n * sizeof(PackJob), cudaMemcpyHostToDevice, st));
    const int threads = 256;
    const int blocks = static_cast<int>((n * 32 + threads - 1) / threads);
    pack_rows_kernel<<<blocks, threads, 0, st>>>(d_jobs, static_cast<int>(n), dst, row_bytes, chunk_bytes, nkc, cw,
                                                 tile_row);
    XLPK_CUDA(cudaGetLastError());
    if (fp8) {
      const long long nt = static_cast<long long>(n) * nkc;
      pack_scales_kernel<<<static_cast<int>((nt + threads - 1) / threads), threads, 0, st>>>(
          d_jobs, static_cast<int>(n), dst, nkc, KC, cw, tile_row);
      XLPK_CUDA(cudaGetLastError());
    } else if (fp4) {
      const long long nt = static_cast<long long>(n) * nkc;
      pack_scales4_kernel<<<static_cast<int>((nt + threads - 1) / threads), threads, 0, st>>>(
          d_jobs, static_cast<int>(n), dst, nkc, KC, cw, tile_row);
      XLPK_CUDA(cudaGetLastError());
    }
    XLPK_CUDA(cudaStreamSynchronize(st));
  }
  out->packed = dst;
  out->gsc = nullptr;
  out->N = N;
  out->K = K;
  out->KC = KC;
  out->fp8 = fp8 ? 1 : 0;
  out->fp4 = fp4 ? 1 : 0;
  if (fp4) {
    // the rows' matrix scales per row pair, behind the packed rows (16-byte aligned)
    std::vector<float> gs(static_cast<size_t>(N));
    for (long long n = 0; n < N; ++n) gs[n] = source_row(ms, n, K, esz, e->cfg, true).g;
    float* d = reinterpret_cast<float*>(dst + align_up(static_cast<size_t>(N) * full_row, 16));
    XLPK_CUDA(cudaMemcpyAsync(d, gs.data(), gs.size() * sizeof(float), cudaMemcpyHostToDevice, st));
    XLPK_CUDA(cudaStreamSynchronize(st));
    out->gsc = reinterpret_cast<const float2*>(d);
  }
  return XLPK_OK;
}

xlpk_status pack_matrix_tc(xlpk_engine* e, const MatSrc& ms, int N, int K, uint8_t* dst, Mat* out,
                           TcRowJob* d_jobs, size_t max_jobs, cudaStream_t st, int win_cols) {
  const int esz = e->esz;
  const bool fp8 = esz == 1;
  const int bc = tc_box_cols(fp8 ? 1 : 0);
  if (N % 8 || K % bc || (win_cols > 0 && (win_cols % bc || win_cols >= K))) return XLPK_ERR_UNSUPPORTED;
  if (fp8 && (!ms.sa || (ms.kind != MatKind::PLAIN && !ms.sb) || (ms.kind == MatKind::QKV && !ms.sc)))
    return XLPK_ERR_INVALID_ARG;
  std::vector<TcRowJob> jobs(static_cast<size_t>(N));
  for (int n = 0; n < N; ++n) {
    const SrcRow sr = source_row(ms, n, K, esz, e->cfg);
    jobs[n] = TcRowJob{sr.w, static_cast<const float*>(sr.s), n};
  }
  const TcGeom g{N, K, e->G, win_cols, fp8 ? 1 : 0};
  for (size_t off = 0; off < jobs.size(); off += max_jobs) {
    const size_t n = std::min(max_jobs, jobs.size() - off);
    XLPK_CUDA(cudaMemcpyAsync(d_jobs, jobs.data() + off, n * sizeof(TcRowJob), cudaMemcpyHostToDevice, st));
    const int threads = 256;
    pack_tc_rows_kernel<<<static_cast<int>((n * 32 + threads - 1) / threads), threads, 0, st>>>(
        d_jobs, static_cast<int>(n), dst, g);
    XLPK_CUDA(cudaGetLastError());
    if (fp8) {
      const long long nt = static_cast<long long>(n) * (K / 128);
      pack_tc_scales_kernel<<<static_cast<int>((nt + threads - 1) / threads), threads, 0, st>>>(
          d_jobs, static_cast<int>(n), dst, g);
      XLPK_CUDA(cudaGetLastError());
    }
    XLPK_CUDA(cudaStreamSynchronize(st));
  }
  out->packed = dst;
  out->gsc = nullptr;
  out->N = N;
  out->K = K;
  out->KC = bc;
  out->fp8 = fp8 ? 1 : 0;
  return XLPK_OK;
}


// Tensor map of one KV cache viewed as a 2-D [rows][d] bf16 array, read in
// boxes of 64 columns x P rows with 128-byte swizzle (the layout the attention
// tile's ldmatrix addressing expects).  The encoder is the driver's
// cuTensorMapEncodeTiled, reached through the runtime's entry-point query so
// the library does not link libcuda.
// bf16 cache: boxes of 64 elements x P rows with the 128-byte swizzle (d/64
// boxes per chunk).  e4m3 cache: one box of d bytes x P rows per chunk with the
// 128-byte (d = 128) or 64-byte (d = 64) swizzle.
xlpk_status encode_kv_map(CUtensorMap* map, void* base, unsigned long long rows, int d, int P, bool fp8 = false) {
  static PFN_cuTensorMapEncodeTiled encode = nullptr;
  if (!encode) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
    if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn) {
      g_cuda_err = "cuTensorMapEncodeTiled unavailable";
      return XLPK_ERR_CUDA;
    }
    encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled>(fn);
  }
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(d) * (fp8 ? 1 : 2)};
  const cuuint32_t box[2] = {fp8 ? static_cast<cuuint32_t>(d) : 64u, static_cast<cuuint32_t>(P)};
  const cuuint32_t estr[2] = {1u, 1u};
  const CUtensorMapSwizzle sw = (fp8 && d == 64) ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
  const CUresult r = encode(map, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base,
                            dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    g_cuda_err = "cuTensorMapEncodeTiled failed (" + std::to_string(static_cast<int>(r)) + ")";
    return XLPK_ERR_CUDA;
  }
  return XLPK_OK;
}

xlpk_status validate_config(const xlpk_config* c) {
  if (!c) return XLPK_ERR_INVALID_ARG;
  if (c->n_layers < 1 || c->n_layers > 1024 || c->hidden <= 0 || c->n_q_heads <= 0 ||
      c->n_kv_heads <= 0 || c->head_dim <= 0 || c->vocab <= 1 || c->batch < 1 || c->max_seq < 1)
    return XLPK_ERR_INVALID_ARG;
  if (c->n_q_heads % c->n_kv_heads != 0) return XLPK_ERR_INVALID_ARG;
  if (c->weight_dtype != XLPK_DTYPE_BF16 && c->weight_dtype != XLPK_DTYPE_FP8_E4M3 &&
      c->weight_dtype != XLPK_DTYPE_NVFP4)
    return XLPK_ERR_INVALID_ARG;
  if (!(c->rms_eps >= 0.f) || !(c->rope_theta > 0.f)) return XLPK_ERR_INVALID_ARG;
  if (c->n_ctas < 0 || c->spin_limit_us < 0) return XLPK_ERR_INVALID_ARG;
  if (c->kv_dtype != XLPK_DTYPE_BF16 && c->kv_dtype != XLPK_DTYPE_FP8_E4M3) return XLPK_ERR_INVALID_ARG;
  if (c->kv_dtype == XLPK_DTYPE_FP8_E4M3) {
    // the scales are powers of two in [2^-24, 2^24]: every rescale is exact
    for (const float sc : {c->k_scale, c->v_scale}) {
      int ex = 0;
      if (!(sc > 0.f) || !std::isfinite(sc) || std::frexp(sc, &ex) != 0.5f || ex - 1 < -24 || ex - 1 > 24)
        return XLPK_ERR_INVALID_ARG;
    }
  }
  if (c->n_experts < 0 || c->top_k < 0 || c->n_shared_experts < 0 || c->expert_ffn < 0)
    return XLPK_ERR_INVALID_ARG;
  // shapes this build handles
  if (c->head_dim != 64 && c->head_dim != 128) return XLPK_ERR_UNSUPPORTED;
  if (c->n_q_heads / c->n_kv_heads > kMaxGroup) return XLPK_ERR_UNSUPPORTED;
  if (c->batch != 1 && c->batch != 2 && c->batch != 4 && c->batch != 8) return XLPK_ERR_UNSUPPORTED;
  if (c->weight_dtype == XLPK_DTYPE_FP8_E4M3) {
    // 128x128 scale blocks tile every matrix exactly
    const int qd = c->n_q_heads * c->head_dim, kvd = c->n_kv_heads * c->head_dim;
    if (c->n_experts > 0) return XLPK_ERR_UNSUPPORTED;
    if (c->hidden % 128 || qd % 128 || kvd % 128 || c->ffn % 128 || c->vocab % 128) return XLPK_ERR_UNSUPPORTED;
    // a packed FP8 row pair over K columns takes 2K + K/16 bytes; bulk copies
    // of row-pair spans need 16-byte multiples, so every K is a multiple of 256
    if (c->hidden % 256 || qd % 256 || c->ffn % 256) return XLPK_ERR_UNSUPPORTED;
  }
  if (c->weight_dtype == XLPK_DTYPE_NVFP4) {
    // dense models at batch 1; K dims in whole 128-column chunks
    const int qd = c->n_q_heads * c->head_dim;
    if (c->n_experts > 0 || c->batch != 1) return XLPK_ERR_UNSUPPORTED;
    if (c->hidden % 128 || qd % 128 || c->ffn % 128) return XLPK_ERR_UNSUPPORTED;
  }
  if (c->n_experts > 0) {
    if (c->top_k < 1 || c->top_k > c->n_experts || c->expert_ffn <= 0) return XLPK_ERR_INVALID_ARG;
    if (c->n_experts > kMaxExperts || c->top_k + c->n_shared_experts > kMaxMoeSlots || c->n_experts % 2)
      return XLPK_ERR_UNSUPPORTED;
    if (c->expert_ffn % 16) return XLPK_ERR_UNSUPPORTED;
    if (c->batch != 1) return XLPK_ERR_UNSUPPORTED;   // per-sequence routing at B > 1 is not built
  } else {
    if (c->top_k != 0 || c->n_shared_experts != 0) return XLPK_ERR_INVALID_ARG;
    if (c->ffn <= 0) return XLPK_ERR_INVALID_ARG;
    if (c->ffn % 16) return XLPK_ERR_UNSUPPORTED;
  }
  if (c->hidden % 16 || (c->n_q_heads * c->head_dim) % 16 || c->vocab % 2) return XLPK_ERR_UNSUPPORTED;
  return XLPK_OK;
}

xlpk_status validate_weights(const xlpk_config* c, const xlpk_weights* w, const xlpk_kv* kv) {
  if (!w || !kv || !w->layers || !w->embed_dev || !w->final_norm_dev || !w->lm_head.w_dev)
    return XLPK_ERR_INVALID_ARG;
  if (!kv->k_dev || !kv->v_dev || !aligned16(kv->k_dev) || !aligned16(kv->v_dev))
    return XLPK_ERR_INVALID_ARG;
  if (kv->page_table_dev) {
    if ((reinterpret_cast<uintptr_t>(kv->page_table_dev) & 3u) || kv->page_size <= 0 || kv->n_pages <= 0)
      return XLPK_ERR_INVALID_ARG;
    // a page is one attention chunk (kTileBytes / 2 of K per chunk)
    // (the same positions for an e4m3 cache: its page is half the bytes)
    if (kv->page_size != (kTileBytes / 2) / (c->head_dim * 2)) return XLPK_ERR_UNSUPPORTED;
  } else if (kv->page_size != 0 || kv->n_pages != 0) {
    return XLPK_ERR_INVALID_ARG;
  }
  if (!aligned16(w->embed_dev) || !aligned16(w->lm_head.w_dev)) return XLPK_ERR_INVALID_ARG;
  if (c->weight_dtype == XLPK_DTYPE_FP8_E4M3) {
    // every linear weight carries its block scales
    if (!w->lm_head.scale_dev) return XLPK_ERR_INVALID_ARG;
    for (int l = 0; l < c->n_layers; ++l) {
      const xlpk_layer_weights& L = w->layers[l];
      const xlpk_linear* lin[] = {&L.wq, &L.wk, &L.wv, &L.wo, &L.w_gate, &L.w_up, &L.w_down};
      for (const xlpk_linear* x : lin)
        if (!x->scale_dev || (reinterpret_cast<uintptr_t>(x->scale_dev) & 3u)) return XLPK_ERR_INVALID_ARG;
    }
  }
  if (c->weight_dtype == XLPK_DTYPE_NVFP4) {
    // every linear weight carries its block scales and a finite positive matrix scale
    auto bad = [](const xlpk_linear& x) {
      return !x.scale_dev || !(x.global_scale > 0.f) || !std::isfinite(x.global_scale);
    };
    if (bad(w->lm_head)) return XLPK_ERR_INVALID_ARG;
    for (int l = 0; l < c->n_layers; ++l) {
      const xlpk_layer_weights& L = w->layers[l];
      for (const xlpk_linear* x : {&L.wq, &L.wk, &L.wv, &L.wo, &L.w_gate, &L.w_up, &L.w_down})
        if (bad(*x)) return XLPK_ERR_INVALID_ARG;
    }
  }
  for (int l = 0; l < c->n_layers; ++l) {
    const xlpk_layer_weights& L = w->layers[l];
    const void* need[] = {L.attn_norm_dev, L.ffn_norm_dev, L.wq.w_dev, L.wk.w_dev, L.wv.w_dev,
                          L.wo.w_dev};
    for (const void* q : need)
      if (!q || !aligned16(q)) return XLPK_ERR_INVALID_ARG;
    if (c->n_experts > 0) {
      const void* moe[] = {L.router_dev, L.we_gate.w_dev, L.we_up.w_dev, L.we_down.w_dev};
      for (const void* q : moe)
        if (!q || !aligned16(q)) return XLPK_ERR_INVALID_ARG;
      if (c->n_shared_experts > 0) {
        const void* sh[] = {L.ws_gate.w_dev, L.ws_up.w_dev, L.ws_down.w_dev};
        for (const void* q : sh)
          if (!q || !aligned16(q)) return XLPK_ERR_INVALID_ARG;
      }
    } else {
      const void* ffn[] = {L.w_gate.w_dev, L.w_up.w_dev, L.w_down.w_dev};
      for (const void* q : ffn)
        if (!q || !aligned16(q)) return XLPK_ERR_INVALID_ARG;
    }
  }
  return XLPK_OK;
}

void fill_rope(std::vector<float2>& t, int max_seq, int d, double theta) {
  const int half = d / 2;
  t.resize(static_cast<size_t>(max_seq) * half);
  for (int pos = 0; pos < max_seq; ++pos)
    for (int i = 0; i < half; ++i) {
      const double inv = std::pow(theta, -2.0 * i / d);
      const double a = static_cast<double>(pos) * inv;
      t[static_cast<size_t>(pos) * half + i] =
          make_float2(static_cast<float>(std::cos(a)), static_cast<float>(std::sin(a)));
    }
}

void free_engine(xlpk_engine* e) {
  if (!e) return;
  if (e->serve_ctl) cudaFreeHost(e->serve_ctl);
  if (e->serve_tokens) cudaFreeHost(e->serve_tokens);
  cudaFree(e->packed);
  cudaFree(e->ws);
  cudaFree(e->d_layers);
  cudaFree(e->rope);
  delete e;
}

xlpk_status create_impl(const xlpk_config* cfg, const xlpk_weights* w, const xlpk_kv* kv,
                        xlpk_engine* e) {
  const xlpk_config& c = *cfg;
  e->cfg = c;
  XLPK_CUDA(cudaGetDevice(&e->device));
  // The weights may still be in flight on any stream of the caller (the
  // packing below runs on a stream of its own that does not wait for them):
  // finish all enqueued work on the device first.
  XLPK_CUDA(cudaDeviceSynchronize());
  cudaDeviceProp prop;
  XLPK_CUDA(cudaGetDeviceProperties(&prop, e->device));
  if (prop.major != 10) {
    g_cuda_err = "device is not sm_100";
    return XLPK_ERR_UNSUPPORTED;
  }
  if (!prop.cooperativeLaunch) return XLPK_ERR_UNSUPPORTED;
  e->G = c.n_ctas > 0 ? c.n_ctas : prop.multiProcessorCount;
  if (e->G > kMaxCtas) {
    g_cuda_err = "persistent grid larger than " + std::to_string(kMaxCtas) + " CTAs";
    return XLPK_ERR_UNSUPPORTED;
  }
  e->esz = c.weight_dtype == XLPK_DTYPE_BF16 ? 2 : 1;
  e->fp4 = c.weight_dtype == XLPK_DTYPE_NVFP4;
  const int B = c.batch, H = c.hidden, d = c.head_dim, F = c.ffn;
  const int qd = c.n_q_heads * d, kvd = c.n_kv_heads * d;
  const int group = c.n_q_heads / c.n_kv_heads;
  e->P = (kTileBytes / 2) / (d * 2);

  // Fused FFN stage (gate/up and a split-K down projection in one stage): bf16
  // dense layers whose output rows fit two 8-row vectors per consumer thread
  // and whose accumulators fit the register budget (XLPK_FFN_FUSED=0 turns it off).
  {
    const bool off = (c.flags & XLPK_FLAG_NO_FUSED_FFN) != 0;
    e->ffn_fused = !off && c.n_experts == 0 && e->esz == 2 && H <= 2 * 8 * kConsumerThreads && H % 8 == 0 &&
                   B <= 2;
  }
  // Batch 8, dense layers: every projection runs on tcgen05 MMAs (8-row units
  // per CTA, M-tiles of <= 128 rows with kTcAccCols accumulator columns each in
  // tensor memory; XLPK_FLAG_NO_TENSOR_CORES keeps the CUDA-core tiles).
  {
    const int bc = e->esz == 1 ? 128 : 64;
    const int nqkv = qd + 2 * kvd;
    e->tc = !(c.flags & XLPK_FLAG_NO_TENSOR_CORES) && B == 8 && c.n_experts == 0 && H % bc == 0 &&
            qd % bc == 0 && F % bc == 0 && nqkv % 8 == 0 && c.vocab % 8 == 0;
    if (e->tc) {
      int mt = 0;
      for (const int n : {nqkv, H, 2 * F, c.vocab}) {
        const int rows = 8 * ((n / 8 + e->G - 1) / e->G);
        mt = std::max(mt, (rows + 127) / 128);
      }
      int cols = 32;
      while (cols < kTcAccCols * mt) cols <<= 1;
      if (cols > 512) e->tc = false;
      e->tc_cols = cols;
    }
  }
  // epilogue side region: RoPE rows, then this CTA's rows of the residual (two
  // planes of float4) and of the embedding (bf16, 8-aligned) for the stages
  // with H output rows, then (fused FFN) the CTA's h slice
  {
    const int maxp = (H / 2 + e->G - 1) / e->G;
    const int rows_max = std::max(2 * maxp, e->tc ? 8 * ((H / 8 + e->G - 1) / e->G) : 0);
    e->side_rope = 0;
    e->side_resid = static_cast<int>(align_up(static_cast<size_t>(B) * d * 4, 16));
    e->nvr = rows_max / 8 + 2;
    e->rows_side = rows_max;
    // the residual rows: two planes of float4, or (fused FFN) int64 rows of the accumulator
    e->side_embed = e->side_resid + B * std::max(2 * e->nvr * 16, rows_max * 8);
    e->evb = static_cast<int>(align_up(static_cast<size_t>(rows_max + 16) * 2, 16));
    e->side_hloc = static_cast<int>(align_up(static_cast<size_t>(e->side_embed) + B * e->evb, 16));
    e->hloc = e->ffn_fused ? (F + e->G - 1) / e->G : 0;
    e->side_bytes = static_cast<int>(align_up(static_cast<size_t>(e->side_hloc) + sizeof(float) * B * e->hloc, 128));
  }
  // shared memory: ring + activation/scratch + control
  const int S_moe = c.n_experts > 0 ? c.top_k + c.n_shared_experts : 0;
  const int attn_scratch = attn_scratch_floats(d, e->G) * 4;
  const int norm_stage = (B + 1) * H * 4;   // normed input vector + its RMSNorm gains
  const int max_smem = static_cast<int>(prop.sharedMemPerBlockOptin);
  auto slots_for = [&](int act) { return (max_smem - act - e->side_bytes - kMiscSmem) / kSlotBytes; };
  e->down_win = 0;
  e->tc_win = 0;
  if (e->tc) {
    // The MMA's B operand takes 32 bytes per input column (8 sequences, a bf16
    // high and low part each).  Projections whose K is larger than a window
    // stream it window by window (tc_window), the window chosen so that the
    // ring keeps at least 4 slots: the whole K, else 4096, 2048 or 1024 columns
    // (whole boxes of either weight type); xlpk_config::window asks for one.
    const int kall = std::max(std::max(H, qd), F);
    auto act_tc = [&](int kw) { return static_cast<int>(align_up(std::max(32 * kw, attn_scratch), 1024)); };
    int win = -1;
    if (c.window > 0) {
      if (c.window % 1024) return XLPK_ERR_UNSUPPORTED;
      win = c.window < kall ? c.window : 0;
    } else {
      for (const int cand : {0, 4096, 2048, 1024}) {
        const int kw = cand > 0 ? std::min(cand, kall) : kall;
        if (slots_for(act_tc(kw)) >= 4) {
          win = cand > 0 && cand < kall ? cand : 0;
          break;
        }
      }
      if (win < 0) win = 1024;
    }
    e->tc_win = win;
    e->act_bytes = act_tc(win > 0 ? win : kall);
  } else {
    auto act_for = [&](int kmax) {
      return static_cast<int>(align_up(std::max(std::max(B * kmax * 4, norm_stage), attn_scratch), 1024));
    };
    e->act_bytes = act_for(std::max(std::max(H, qd), std::max(F, S_moe * c.expert_ffn)));
    // the fused-FFN layers stage their int64 residual behind the fp32 input
    if (e->ffn_fused) e->act_bytes = std::max(e->act_bytes, static_cast<int>(align_up(static_cast<size_t>(12) * B * H, 1024)));
    // A two-stage dense FFN whose down-projection input (B x F fp32) would leave
    // the ring fewer than 3 slots streams W_down window by window instead: the
    // activation region then holds B x down_win floats of h at a time (windows
    // of the largest whole number of k-chunks that fits the other stages'
    // inputs; xlpk_config::window asks for a given window where windows are
    // possible).
    const int kc = pick_kc(F, e->esz);
    const int maxp = (H / 2 + e->G - 1) / e->G;
    const bool possible =
        !e->ffn_fused && c.n_experts == 0 && B >= 2 && kc > 0 && maxp <= kPairsPerTile * kMaxWinGroups;
    int win = 0;
    if (possible && c.window > 0) {
      if (c.window % kc == 0 && c.window < F) win = c.window;
    } else if (possible && F > std::max(H, qd) && slots_for(e->act_bytes) < 3) {
      win = (std::max(H, qd) / kc) * kc;
      if (win >= F) win = 0;
    }
    if (win > 0) {
      e->down_win = win;
      e->act_bytes = act_for(std::max(std::max(H, qd), win));
    }
  }
  e->shallow = B <= 4;
  e->nslot = std::min(e->shallow ? kShallowSlots : kMaxSlots,
                      (max_smem - e->act_bytes - e->side_bytes - kMiscSmem) / kSlotBytes);
  if (e->nslot < 2) return XLPK_ERR_UNSUPPORTED;
  e->smem = e->nslot * kSlotBytes + e->act_bytes + e->side_bytes + kMiscSmem;
  const int var = (c.kv_dtype == XLPK_DTYPE_FP8_E4M3 ? 1 : 0) | (e->fp4 ? 2 : 0);
  if (!bind_by_shape(e, B, d, c.n_experts > 0, var)) return XLPK_ERR_UNSUPPORTED;

  // The attribute is per kernel function, shared by every handle that uses the
  // same instantiation: allow the device maximum rather than this handle's size.
  XLPK_CUDA(cudaFuncSetAttribute(e->kern_persistent, cudaFuncAttributeMaxDynamicSharedMemorySize, max_smem));
  XLPK_CUDA(cudaFuncSetAttribute(e->kern_stage, cudaFuncAttributeMaxDynamicSharedMemorySize, max_smem));
  int per_sm = 0;
  XLPK_CUDA(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, e->kern_persistent, kThreads, e->smem));
  if (per_sm < 1 || e->G > per_sm * prop.multiProcessorCount) {
    g_cuda_err = "persistent grid does not fit co-resident";
    return XLPK_ERR_UNSUPPORTED;
  }

  // packed weights: per layer qkv, o, then gate/up + down (dense) or the
  // router + every expert's gate/up and down (MoE); then the LM head
  enum Role { R_QKV, R_O, R_GU, R_DOWN, R_DOWNT, R_ROUTER, R_EGU, R_EDOWN, R_LM };
  struct MatPlan {
    MatSrc src;
    int N, K;
    size_t off;
    int layer, role, split;
  };
  const bool moe = c.n_experts > 0;
  const int Fe = c.expert_ffn, nE = c.n_experts + c.n_shared_experts;
  std::vector<MatPlan> mats;
  size_t total = 0;
  auto add = [&](MatSrc s, int N, int K, int layer, int role, int split) {
    mats.push_back({s, N, K, total, layer, role, split});
    const size_t esz_m = role == R_ROUTER ? 2 : e->esz;
    const size_t nk = static_cast<size_t>(N) * K;
    if (e->fp4 && role != R_ROUTER)   // codes + e4m3 block scales, then the per-row matrix scales
      total += align_up(align_up(nk / 2 + nk / 16, 16) + static_cast<size_t>(N) * 4, 256);
    else
      total += align_up(nk * esz_m + (esz_m == 1 ? nk / 32 : 0), 256);
  };
  auto u8 = [](const void* p) { return static_cast<const uint8_t*>(p); };
  const size_t eg_bytes = static_cast<size_t>(Fe) * H * e->esz;   // one expert's gate (or up, or down)
  for (int l = 0; l < c.n_layers; ++l) {
    const xlpk_layer_weights& L = w->layers[l];
    add({MatKind::QKV, u8(L.wq.w_dev), u8(L.wk.w_dev), u8(L.wv.w_dev), L.wq.scale_dev, L.wk.scale_dev,
         L.wv.scale_dev, L.wq.global_scale, L.wk.global_scale, L.wv.global_scale},
        qd + 2 * kvd, H, l, R_QKV, e->G);
    add({MatKind::PLAIN, u8(L.wo.w_dev), nullptr, nullptr, L.wo.scale_dev, nullptr, nullptr, L.wo.global_scale}, H,
        qd, l, R_O, e->G);
    if (!moe) {
      add({MatKind::GATEUP, u8(L.w_gate.w_dev), u8(L.w_up.w_dev), nullptr, L.w_gate.scale_dev, L.w_up.scale_dev,
           nullptr, L.w_gate.global_scale, L.w_up.global_scale},
          2 * F, H, l, R_GU, e->G);
      if (e->ffn_fused)
        add({MatKind::PLAIN, u8(L.w_down.w_dev), nullptr, nullptr}, F, H, l, R_DOWNT, 1);   // W_down^T [F][H]
      else
        add({MatKind::PLAIN, u8(L.w_down.w_dev), nullptr, nullptr, L.w_down.scale_dev, nullptr, nullptr,
             L.w_down.global_scale},
            H, F, l, R_DOWN, e->G);
    } else {
      // router logits are bf16 whatever the weight dtype
      add({MatKind::PLAIN, u8(L.router_dev), nullptr, nullptr}, c.n_experts, H, l, R_ROUTER, 1);
      for (int x = 0; x < nE; ++x) {
        const bool sh = x >= c.n_experts;
        const int xi = sh ? x - c.n_experts : x;
        const uint8_t* g = u8(sh ? L.ws_gate.w_dev : L.we_gate.w_dev) + xi * eg_bytes;
        const uint8_t* u = u8(sh ? L.ws_up.w_dev : L.we_up.w_dev) + xi * eg_bytes;
        add({MatKind::GATEUP, g, u, nullptr}, 2 * Fe, H, l, R_EGU, 1);
      }
      for (int x = 0; x < nE; ++x) {
        const bool sh = x >= c.n_experts;
        const int xi = sh ? x - c.n_experts : x;
        const uint8_t* dn = u8(sh ? L.ws_down.w_dev : L.we_down.w_dev) + xi * eg_bytes;
        add({MatKind::PLAIN, dn, nullptr, nullptr}, H, Fe, l, R_EDOWN, e->G);
      }
    }
  }
  add({MatKind::PLAIN, u8(w->lm_head.w_dev), nullptr, nullptr, w->lm_head.scale_dev, nullptr, nullptr,
       w->lm_head.global_scale},
      c.vocab, H, -1, R_LM, e->G);
  // library-owned copies of the embedding table and the norm gains, so the
  // caller may free every weight buffer after create
  const size_t off_embed = total;
  total += align_up(static_cast<size_t>(c.vocab) * H * 2, 256);
  const size_t off_norms = total;
  total += align_up(sizeof(float) * H * (2 * static_cast<size_t>(c.n_layers) + 1), 256);
  e->packed_bytes = total;
  XLPK_CUDA(cudaMalloc(&e->packed, total));
#ifdef XLPK_DEBUG_POISON
  XLPK_CUDA(cudaMemset(e->packed, 0xff, total));   // debug build: unwritten bytes read as NaN
#endif
  // weights streamed per step: every dense matrix; for MoE the router and the
  // shared + top_k experts of each layer
  e->weight_bytes_per_step = 0;
  for (const MatPlan& m : mats) {
    if (m.role == R_EGU || m.role == R_EDOWN) continue;
    const int64_t nk = static_cast<int64_t>(m.N) * m.K;
    e->weight_bytes_per_step += m.role == R_ROUTER ? 2 * nk
                                : e->fp4       ? nk / 2 + nk / 16 + 4
                                : e->esz == 1  ? nk + nk / 32
                                               : 2 * nk;
  }
  if (moe)
    e->weight_bytes_per_step += static_cast<int64_t>(c.n_layers) * (c.top_k + c.n_shared_experts) * 3 *
                                static_cast<int64_t>(eg_bytes);

  cudaStream_t st;
  XLPK_CUDA(cudaStreamCreateWithFlags(&st, cudaStreamNonBlocking));
  const size_t max_jobs = 1 << 20;
  PackJob* d_jobs = nullptr;
  cudaError_t ce = cudaMalloc(&d_jobs, max_jobs * sizeof(PackJob));
  if (ce != cudaSuccess) {
    cudaStreamDestroy(st);
    return cuda_fail(ce, "cudaMalloc(jobs)");
  }
  std::vector<LayerParams> lp(c.n_layers);
  Mat lm{};
  xlpk_status rc = XLPK_OK;
  const int esz_saved = e->esz;
  for (size_t i = 0; i < mats.size() && rc == XLPK_OK; ++i) {
    const MatPlan& mp = mats[i];
    Mat m{};
    if (mp.role == R_DOWNT) {
      // the fused FFN streams W_down columns: store W_down^T, plain bf16 [F][H]
      const dim3 tb(32, 8), gr((mp.N + 31) / 32, (mp.K + 31) / 32);   // in: [H=K][F=N]
      transpose_bf16_kernel<<<gr, tb, 0, st>>>(reinterpret_cast<const uint16_t*>(mp.src.a),
                                               reinterpret_cast<uint16_t*>(e->packed + mp.off), mp.K, mp.N);
      ce = cudaGetLastError();
      if (ce == cudaSuccess) ce = cudaStreamSynchronize(st);
      if (ce != cudaSuccess) {
        rc = cuda_fail(ce, "transpose_bf16_kernel");
        break;
      }
      m.packed = e->packed + mp.off;
      m.N = mp.N;
      m.K = mp.K;
      m.KC = mp.K;
      m.fp8 = 0;
    } else {
      e->esz = mp.role == R_ROUTER ? 2 : esz_saved;
      if (e->tc && (mp.role == R_QKV || mp.role == R_O || mp.role == R_GU || mp.role == R_DOWN || mp.role == R_LM))
        rc = pack_matrix_tc(e, mp.src, mp.N, mp.K, e->packed + mp.off, &m, reinterpret_cast<TcRowJob*>(d_jobs),
                            max_jobs, st, tc_window(e->tc_win, mp.K));
      else
        rc = pack_matrix(e, mp.src, mp.N, mp.K, e->packed + mp.off, &m, d_jobs, max_jobs, st, mp.split,
                         mp.role == R_DOWN ? e->down_win : 0);
      e->esz = esz_saved;
    }
    if (rc != XLPK_OK) break;
    LayerParams* L = mp.layer >= 0 ? &lp[mp.layer] : nullptr;
    switch (mp.role) {
      case R_QKV: L->qkv = m; break;
      case R_O: L->o = m; break;
      case R_GU: L->gu = m; break;
      case R_DOWN: L->down = m; break;
      case R_DOWNT: L->downT = m; break;
      case R_ROUTER: L->router = m; break;
      case R_EGU:
        if (!L->egu.packed) L->egu = m;
        L->egu_stride = static_cast<long long>(align_up(2 * eg_bytes, 256));
        break;
      case R_EDOWN:
        if (!L->edown.packed) L->edown = m;
        L->edown_stride = static_cast<long long>(align_up(eg_bytes, 256));
        break;
      default: lm = m; break;
    }
  }
  cudaFree(d_jobs);
  cudaStreamDestroy(st);
  if (rc != XLPK_OK) return rc;
  uint16_t* embed_copy = reinterpret_cast<uint16_t*>(e->packed + off_embed);
  float* norms = reinterpret_cast<float*>(e->packed + off_norms);
  XLPK_CUDA(cudaMemcpy(embed_copy, w->embed_dev, static_cast<size_t>(c.vocab) * H * 2, cudaMemcpyDeviceToDevice));
  for (int l = 0; l < c.n_layers; ++l) {
    float* an = norms + static_cast<size_t>(2 * l) * H;
    float* fn = an + H;
    XLPK_CUDA(cudaMemcpy(an, w->layers[l].attn_norm_dev, sizeof(float) * H, cudaMemcpyDeviceToDevice));
    XLPK_CUDA(cudaMemcpy(fn, w->layers[l].ffn_norm_dev, sizeof(float) * H, cudaMemcpyDeviceToDevice));
    lp[l].attn_norm = an;
    lp[l].ffn_norm = fn;
  }
  float* final_norm_copy = norms + static_cast<size_t>(2 * c.n_layers) * H;
  XLPK_CUDA(cudaMemcpy(final_norm_copy, w->final_norm_dev, sizeof(float) * H, cudaMemcpyDeviceToDevice));
  XLPK_CUDA(cudaMalloc(&e->d_layers, sizeof(LayerParams) * c.n_layers));
  XLPK_CUDA(cudaMemcpy(e->d_layers, lp.data(), sizeof(LayerParams) * c.n_layers, cudaMemcpyHostToDevice));

  std::vector<float2> rope;
  fill_rope(rope, c.max_seq, d, c.rope_theta);
  XLPK_CUDA(cudaMalloc(&e->rope, rope.size() * sizeof(float2)));
  XLPK_CUDA(cudaMemcpy(e->rope, rope.data(), rope.size() * sizeof(float2), cudaMemcpyHostToDevice));

  // workspace arena with fixed offsets
  // attention partials: one row per (sequence, kv head, contributing CTA)
  const long long prow = static_cast<long long>(B) * c.n_kv_heads * e->G;
  CounterLayout cl;
  cl.lm_arrive = c.n_layers * ST_LAYER;
  cl.step_done = cl.lm_arrive + 1;
  cl.attn_arrive = cl.step_done + 1;
  cl.total = cl.attn_arrive + c.n_layers * B * c.n_kv_heads;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes, 256);
    return o;
  };
  const size_t o_x = take(sizeof(float) * B * H);
  const size_t o_q = take(sizeof(float) * B * qd);
  const size_t o_o = take(sizeof(float) * B * qd);
  const size_t o_h = take(sizeof(float) * B * std::max(F, S_moe * c.expert_ffn));
  const size_t o_y = take(sizeof(float) * B * H);
  const size_t o_xacc = take(sizeof(long long) * B * H);
  const size_t o_pml = take(sizeof(float) * prow * group * 2);
  const size_t o_po = take(sizeof(float) * prow * group * d);
  const size_t o_lv = take(sizeof(float) * e->G * B);
  const size_t o_li = take(sizeof(int) * e->G * B);
  const size_t o_rte = take(sizeof(int) * c.n_layers * std::max(S_moe, 1));
  const size_t o_rtw = take(sizeof(float) * c.n_layers * std::max(S_moe, 1));
  const size_t o_cnt = take(sizeof(unsigned) * cl.total);
  const size_t o_tok = take(sizeof(int) * B);
  const size_t o_st = take(sizeof(int) * 4);
  const size_t o_ab = take(sizeof(int));
  const size_t o_ts = take(sizeof(int) * static_cast<size_t>(c.max_seq) * B);
  const size_t o_sv = take(sizeof(unsigned) * 2);
  const size_t o_acc = take(sizeof(int32_t));
  e->ws_bytes = off;
  XLPK_CUDA(cudaMalloc(&e->ws, e->ws_bytes));
  XLPK_CUDA(cudaMemset(e->ws, 0, e->ws_bytes));
#ifdef XLPK_DEBUG_POISON
  // debug build: scratch that every step must write before reading it holds NaN
  XLPK_CUDA(cudaMemset(e->ws + o_x, 0xff, o_lv - o_x));
#endif

  Params& p = e->base;
  p.L = c.n_layers;
  p.H = H;
  p.nq = c.n_q_heads;
  p.nkv = c.n_kv_heads;
  p.d = d;
  p.F = F;
  p.V = c.vocab;
  p.B = B;
  p.max_seq = c.max_seq;
  p.group = group;
  p.esz = e->esz;
  p.eps = c.rms_eps;
  p.qk_scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(d)));
  p.G = e->G;
  p.nslot = e->nslot;
  p.act_bytes = e->act_bytes;
  p.side_bytes = e->side_bytes;
  p.side_rope = e->side_rope;
  p.side_resid = e->side_resid;
  p.side_embed = e->side_embed;
  p.nvr = e->nvr;
  p.rows_side = e->rows_side;
  p.evb = e->evb;
  p.attn_pos_per_tile = e->P;
  p.spin_limit_ns = 1000LL * (c.spin_limit_us > 0 ? c.spin_limit_us : 200000);
  p.l2_prefetch_bytes = e->shallow ? kShallowPrefetchBytes : kPrefetchBytes;
  p.wait_hint_ns = 20000;
  p.cl = cl;
  p.embed = embed_copy;
  p.final_norm = final_norm_copy;
  p.lm = lm;
  p.layers = e->d_layers;
  const bool kv8 = c.kv_dtype == XLPK_DTYPE_FP8_E4M3;
  p.kv_fp8 = kv8 ? 1 : 0;
  p.kc = kv8 ? nullptr : static_cast<uint16_t*>(kv->k_dev);
  p.vc = kv8 ? nullptr : static_cast<uint16_t*>(kv->v_dev);
  p.kc8 = kv8 ? static_cast<uint8_t*>(kv->k_dev) : nullptr;
  p.vc8 = kv8 ? static_cast<uint8_t*>(kv->v_dev) : nullptr;
  p.k_scale = kv8 ? c.k_scale : 1.f;
  p.v_scale = kv8 ? c.v_scale : 1.f;
  p.k_inv = 1.f / p.k_scale;   // exact: powers of two
  p.v_inv = 1.f / p.v_scale;
  p.page_table = kv->page_table_dev;
  p.n_pages = kv->page_table_dev ? kv->n_pages : 0;
  p.pages_per_seq = (c.max_seq + e->P - 1) / e->P;
  {
    const unsigned long long rows =
        kv->page_table_dev
            ? static_cast<unsigned long long>(c.n_layers) * kv->n_pages * c.n_kv_heads * static_cast<unsigned long long>(e->P)
            : static_cast<unsigned long long>(c.n_layers) * B * c.n_kv_heads * static_cast<unsigned long long>(c.max_seq);
    xlpk_status st = encode_kv_map(&p.tmap_k, kv->k_dev, rows, d, e->P, kv8);
    if (st != XLPK_OK) return st;
    st = encode_kv_map(&p.tmap_v, kv->v_dev, rows, d, e->P, kv8);
    if (st != XLPK_OK) return st;
  }
  p.rope = e->rope;
  p.x = reinterpret_cast<float*>(e->ws + o_x);
  p.q = reinterpret_cast<float*>(e->ws + o_q);
  p.o = reinterpret_cast<float*>(e->ws + o_o);
  p.h = reinterpret_cast<float*>(e->ws + o_h);
  p.y = reinterpret_cast<float*>(e->ws + o_y);
  p.xacc = reinterpret_cast<long long*>(e->ws + o_xacc);
  p.ffn_fused = e->ffn_fused ? 1 : 0;
  p.resid_fixed = e->ffn_fused && !(c.flags & XLPK_FLAG_FLOAT_FFN_REDUCE) ? 1 : 0;
  p.jt = kTileBytes / (H * 2);
  p.down_win = e->down_win;
  p.tc = e->tc ? 1 : 0;
  p.tc_cols = e->tc_cols;
  p.tc_win = e->tc_win;
  p.side_hloc = e->side_hloc;
  p.hloc = e->hloc;
  p.route_exp = reinterpret_cast<int*>(e->ws + o_rte);
  p.route_w = reinterpret_cast<float*>(e->ws + o_rtw);
  p.E = c.n_experts;
  p.topk = c.top_k;
  p.nsh = c.n_shared_experts;
  p.S = S_moe;
  p.Fe = c.expert_ffn;
  p.part_ml = reinterpret_cast<float*>(e->ws + o_pml);
  p.part_o = reinterpret_cast<float*>(e->ws + o_po);
  p.lm_val = reinterpret_cast<float*>(e->ws + o_lv);
  p.lm_idx = reinterpret_cast<int*>(e->ws + o_li);
  p.cnt = reinterpret_cast<unsigned*>(e->ws + o_cnt);
  p.cur_tok = reinterpret_cast<int*>(e->ws + o_tok);
  p.status = reinterpret_cast<int*>(e->ws + o_st);
  p.abort_flag = reinterpret_cast<int*>(e->ws + o_ab);
  e->tok_scratch = reinterpret_cast<int32_t*>(e->ws + o_ts);
  e->serve_dev_words = reinterpret_cast<unsigned*>(e->ws + o_sv);
  e->verify_word = reinterpret_cast<int32_t*>(e->ws + o_acc);
  e->pos.assign(B, 0);
  XLPK_CUDA(cudaDeviceSynchronize());
  return XLPK_OK;
}

xlpk_status check_decode_args(xlpk_engine* h, int32_t n_steps, int32_t* tokens_out) {
  if (!h || n_steps < 0) return XLPK_ERR_INVALID_ARG;
  if (h->serve_active) return XLPK_ERR_INVALID_ARG;   // the serve loop owns the handle
  if (n_steps > 0 && !tokens_out) return XLPK_ERR_INVALID_ARG;
  for (int b = 0; b < h->cfg.batch; ++b)
    if (static_cast<long long>(h->pos[b]) + n_steps > h->cfg.max_seq) return XLPK_ERR_KV_FULL;
  return XLPK_OK;
}

Params call_params(xlpk_engine* h, int32_t n_steps, int32_t* tokens_out, const xlpk_decode_io* io) {
  Params p = h->base;
  p.n_steps = n_steps;
  p.step_base = h->step_base;
  for (int b = 0; b < kMaxBatch; ++b) p.pos0[b] = b < h->cfg.batch ? h->pos[b] : 0;
  p.tokens_out = tokens_out;
  p.forced = io ? io->forced_tokens_dev : nullptr;
  p.logits_out = io ? io->logits_dev : nullptr;
  p.hidden_out = io ? io->hidden_dev : nullptr;
  // parity mode: the registered buffers, each step over the last
  p.logits_overwrite = 0;
  p.hidden_overwrite = 0;
  if (!p.logits_out && h->dbg_logits) {
    p.logits_out = h->dbg_logits;
    p.logits_overwrite = 1;
  }
  if (!p.hidden_out && h->dbg_hidden) {
    p.hidden_out = h->dbg_hidden;
    p.hidden_overwrite = 1;
  }
  p.experts_out = io ? io->experts_dev : nullptr;
  p.trace = io ? reinterpret_cast<unsigned long long*>(io->trace_dev) : nullptr;
  // Failure-detection testing: CTA 0 withholds its release of one stage at the
  // call's first step, so a dependency wait runs out (nothing faults).
  p.fault_drop_stage = io && io->withhold_release > 0 ? io->withhold_release - 1 : -1;
  return p;
}

void advance(xlpk_engine* h, int32_t n_steps, cudaStream_t st) {
  for (int b = 0; b < h->cfg.batch; ++b) h->pos[b] += n_steps;
  h->step_base += n_steps;
  h->last_stream = st;
}

}  // namespace

// ------------------------------------------------------------------ allocation-free decode
// Scratch of xlpk_decode_noalloc: one library-wide array on every device that
// loads the library.  Host code must not use the symbol's host address; the
// device address comes from cudaGetSymbolAddress, once per device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[XLPK_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
unsigned char* g_noalloc_addr[kMaxDevices] = {};
unsigned long long g_noalloc_ctx[kMaxDevices] = {};   // context the address was taken in

// Unique id of the current context (driver entry points reached through the
// runtime, so the library does not link libcuda); 0 if unavailable.
unsigned long long current_context_id() {
  using GetCurrent = CUresult (*)(CUcontext*);
  using GetId = CUresult (*)(CUcontext, unsigned long long*);
  static GetCurrent get_current = nullptr;
  static GetId get_id = nullptr;
  static bool looked_up = false;
  if (!looked_up) {
    looked_up = true;
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<GetCurrent>(f);
    f = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<GetId>(f);
  }
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Device address of the array on `dev` (which must be the current device):
// looked up once per device, and again if the device's context has been
// replaced since (cudaDeviceReset reloads the module, which may move it).
xlpk_status noalloc_scratch(int dev, unsigned char** out) {
  if (dev < 0 || dev >= kMaxDevices) return XLPK_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  const unsigned long long ctx = current_context_id();
  if (!g_noalloc_addr[dev] || ctx != g_noalloc_ctx[dev]) {
    void* ptr = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess || !ptr) return cuda_fail(e, "cudaGetSymbolAddress(g_noalloc_scratch)");
    g_noalloc_addr[dev] = static_cast<unsigned char*>(ptr);
    g_noalloc_ctx[dev] = ctx;
  }
  *out = g_noalloc_addr[dev];
  return XLPK_OK;
}

// ---- serve mode: one persistent launch that stays resident across requests

// Steps of the current serve launch the host has seen completed.
long long serve_done(const xlpk_engine* h) {
  return static_cast<long long>(*reinterpret_cast<const volatile unsigned*>(h->serve_ctl + 2));
}

// Launch the serve loop from the handle's current state (session step serve_step0).
xlpk_status serve_launch(xlpk_engine* h) {
  const xlpk_config& c = h->cfg;
  int room = c.max_seq;
  for (int b = 0; b < c.batch; ++b) room = std::min(room, c.max_seq - h->pos[b]);
  if (room <= 0) return XLPK_ERR_KV_FULL;
  Params p = call_params(h, room, h->tok_scratch, nullptr);
  p.serve = 1;
  p.serve_step0 = static_cast<int>(h->serve_step0);
  p.serve_req_host = h->serve_ctl_dev;
  p.serve_exit_host = reinterpret_cast<const int*>(h->serve_ctl_dev + 1);
  p.serve_done_host = h->serve_ctl_dev + 2;
  p.serve_tokens_host = h->serve_tokens_dev;
  p.serve_cap = h->serve_cap;
  p.serve_req_dev = h->serve_dev_words;
  p.serve_stop_dev = reinterpret_cast<int*>(h->serve_dev_words + 1);
  p.serve_idle_ns = h->serve_idle_ns;
  const unsigned init[2] = {static_cast<unsigned>(h->serve_step0), 0xffffffffu};   // forwarded = done; no stop
  XLPK_CUDA(cudaMemcpyAsync(h->serve_dev_words, init, sizeof(init), cudaMemcpyHostToDevice, h->serve_stream));
  void* args[] = {&p};
  XLPK_CUDA(cudaLaunchCooperativeKernel(h->kern_persistent, dim3(h->G), dim3(kThreads), args,
                                        static_cast<size_t>(h->smem), h->serve_stream));
  h->serve_launched = true;
  h->last_stream = h->serve_stream;
  return XLPK_OK;
}

// The current launch has ended: fold the steps it decoded into the handle's
// state.  Returns the launch's device status.
xlpk_status serve_collect(xlpk_engine* h) {
  XLPK_CUDA(cudaStreamSynchronize(h->serve_stream));
  h->serve_launched = false;
  const long long done = serve_done(h);
  const int n = static_cast<int>(done - h->serve_step0);
  for (int b = 0; b < h->cfg.batch; ++b) h->pos[b] += n;
  h->step_base += n;
  h->serve_step0 = done;
  return xlpk_get_status(h);
}

}  // namespace

extern "C" {

xlpk_status xlpk_serve_start(xlpk_handle h, int32_t idle_limit_us, void* stream) {
  if (!h || idle_limit_us <= 0 || h->serve_active) return XLPK_ERR_INVALID_ARG;
  if (h->cfg.n_experts > 0 && h->cfg.batch != 1) return XLPK_ERR_UNSUPPORTED;
  if (!h->serve_ctl) {
    void* ctl = nullptr;
    void* tok = nullptr;
    XLPK_CUDA(cudaHostAlloc(&ctl, 64, cudaHostAllocMapped));
    h->serve_ctl = static_cast<unsigned*>(ctl);
    h->serve_cap = h->cfg.max_seq;
    XLPK_CUDA(cudaHostAlloc(&tok, sizeof(int32_t) * static_cast<size_t>(h->serve_cap) * h->cfg.batch,
                            cudaHostAllocMapped));
    h->serve_tokens = static_cast<int32_t*>(tok);
    XLPK_CUDA(cudaHostGetDevicePointer(reinterpret_cast<void**>(&h->serve_ctl_dev), h->serve_ctl, 0));
    XLPK_CUDA(cudaHostGetDevicePointer(reinterpret_cast<void**>(&h->serve_tokens_dev), h->serve_tokens, 0));
  }
  volatile unsigned* w = h->serve_ctl;
  w[0] = 0u;
  w[1] = 0u;
  w[2] = 0u;
  h->serve_posted = 0;
  h->serve_step0 = 0;
  h->serve_idle_ns = 1000LL * idle_limit_us;
  h->serve_stream = static_cast<cudaStream_t>(stream);
  h->serve_active = true;
  const xlpk_status rc = serve_launch(h);
  if (rc != XLPK_OK) h->serve_active = false;
  return rc;
}

xlpk_status xlpk_serve_post(xlpk_handle h, int32_t n_steps, int64_t* first_step) {
  if (!h || !h->serve_active || n_steps <= 0 || !first_step) return XLPK_ERR_INVALID_ARG;
  // every step of the session must fit the cache
  const long long pos_start = h->pos[0] - h->serve_step0;   // pos at the session start (sequence 0)
  for (int b = 0; b < h->cfg.batch; ++b)
    if (h->pos[b] - h->serve_step0 + h->serve_posted + n_steps > h->cfg.max_seq) return XLPK_ERR_KV_FULL;
  (void)pos_start;
  if (h->serve_launched && cudaStreamQuery(h->serve_stream) == cudaSuccess) {
    // the loop left while idle: fold in its steps and start it again
    const xlpk_status rc = serve_collect(h);
    if (rc != XLPK_OK) return rc;
  }
  if (!h->serve_launched) {
    const xlpk_status rc = serve_launch(h);
    if (rc != XLPK_OK) return rc;
  }
  *first_step = h->serve_posted;
  h->serve_posted += n_steps;
  std::atomic_thread_fence(std::memory_order_release);
  *reinterpret_cast<volatile unsigned*>(h->serve_ctl) = static_cast<unsigned>(h->serve_posted);
  return XLPK_OK;
}

xlpk_status xlpk_serve_wait(xlpk_handle h, int64_t first_step, int32_t n_steps, int32_t* tokens_out_host,
                            int32_t timeout_us) {
  if (!h || !h->serve_active || n_steps <= 0 || first_step < 0 || !tokens_out_host || timeout_us <= 0)
    return XLPK_ERR_INVALID_ARG;
  const long long target = first_step + n_steps;
  if (target > h->serve_posted) return XLPK_ERR_INVALID_ARG;
  const auto t0 = std::chrono::steady_clock::now();
  auto last_check = t0;
  while (serve_done(h) < target) {
    // whether the loop has left (idle) is asked of the driver only now and then
    const auto now = std::chrono::steady_clock::now();
    if (now - last_check < std::chrono::microseconds(200)) continue;
    last_check = now;
    if (h->serve_launched && cudaStreamQuery(h->serve_stream) == cudaSuccess && serve_done(h) < target) {
      // the launch ended (idle) before our steps: start it again
      xlpk_status rc = serve_collect(h);
      if (rc != XLPK_OK) return rc;
      rc = serve_launch(h);
      if (rc != XLPK_OK) return rc;
    }
    if (std::chrono::duration_cast<std::chrono::microseconds>(std::chrono::steady_clock::now() - t0).count() >
        timeout_us)
      return XLPK_ERR_TIMEOUT;
  }
  std::atomic_thread_fence(std::memory_order_acquire);
  const volatile int32_t* ring = h->serve_tokens;
  const int B = h->cfg.batch;
  for (long long t = first_step; t < target; ++t)
    for (int b = 0; b < B; ++b)
      tokens_out_host[(t - first_step) * B + b] = ring[(t % h->serve_cap) * B + b];
  return XLPK_OK;
}

xlpk_status xlpk_serve_stop(xlpk_handle h) {
  if (!h || !h->serve_active) return XLPK_ERR_INVALID_ARG;
  std::atomic_thread_fence(std::memory_order_release);
  *reinterpret_cast<volatile unsigned*>(h->serve_ctl + 1) = 1u;
  xlpk_status rc = XLPK_OK;
  if (h->serve_launched) rc = serve_collect(h);
  h->serve_active = false;
  return rc;
}


xlpk_status xlpk_create(const xlpk_config* cfg, const xlpk_weights* weights, const xlpk_kv* kv,
                        xlpk_handle* out) {
  if (!out) return XLPK_ERR_INVALID_ARG;
  *out = nullptr;
  xlpk_status rc = validate_config(cfg);
  if (rc != XLPK_OK) return rc;
  rc = validate_weights(cfg, weights, kv);
  if (rc != XLPK_OK) return rc;
  xlpk_engine* e = new xlpk_engine();
  rc = create_impl(cfg, weights, kv, e);
  if (rc != XLPK_OK) {
    free_engine(e);
    return rc;
  }
  *out = e;
  return XLPK_OK;
}

xlpk_status xlpk_destroy(xlpk_handle h) {
  if (!h) return XLPK_ERR_INVALID_ARG;
  cudaDeviceSynchronize();
  free_engine(h);
  return XLPK_OK;
}

xlpk_status xlpk_set_state(xlpk_handle h, const int32_t* tokens_host, const int32_t* seq_lens_host,
                           void* stream) {
  if (!h || !tokens_host || !seq_lens_host) return XLPK_ERR_INVALID_ARG;
  if (h->serve_active) return XLPK_ERR_INVALID_ARG;   // the serve loop owns the handle
  for (int b = 0; b < h->cfg.batch; ++b) {
    if (tokens_host[b] < 0 || tokens_host[b] >= h->cfg.vocab) return XLPK_ERR_INVALID_ARG;
    if (seq_lens_host[b] < 0 || seq_lens_host[b] >= h->cfg.max_seq) return XLPK_ERR_INVALID_ARG;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  XLPK_CUDA(cudaMemcpyAsync(h->base.cur_tok, tokens_host, sizeof(int32_t) * h->cfg.batch,
                            cudaMemcpyHostToDevice, st));
  for (int b = 0; b < h->cfg.batch; ++b) h->pos[b] = seq_lens_host[b];
  h->last_stream = st;
  return XLPK_OK;
}

xlpk_status xlpk_decode(xlpk_handle h, int32_t n_steps, int32_t* tokens_out_dev,
                        const xlpk_decode_io* io, void* stream) {
  xlpk_status rc = check_decode_args(h, n_steps, tokens_out_dev);
  if (rc != XLPK_OK || n_steps == 0) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Params p = call_params(h, n_steps, tokens_out_dev, io);
  void* args[] = {&p};
  XLPK_CUDA(cudaLaunchCooperativeKernel(h->kern_persistent, dim3(h->G), dim3(kThreads), args,
                                        static_cast<size_t>(h->smem), st));
  advance(h, n_steps, st);
  return XLPK_OK;
}

xlpk_status xlpk_decode_unfused(xlpk_handle h, int32_t n_steps, int32_t* tokens_out_dev,
                                const xlpk_decode_io* io, void* stream) {
  xlpk_status rc = check_decode_args(h, n_steps, tokens_out_dev);
  if (rc != XLPK_OK || n_steps == 0) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Params p = call_params(h, n_steps, tokens_out_dev, io);
  // Fresh dependency counters for every call (the last-arriver decisions count
  // from step 0), so the launches this call records can be captured into a CUDA
  // graph and replayed; a later persistent call continues from step n_steps.
  XLPK_CUDA(cudaMemsetAsync(h->base.cnt, 0, sizeof(unsigned) * h->base.cl.total, st));
  p.step_base = 0;
  for (int s = 0; s < n_steps; ++s) {
    for (int l = 0; l < h->cfg.n_layers; ++l)
      for (int k = 0; k < ST_LAYER; ++k)
        if (!(k == ST_DOWN && h->ffn_fused)) h->launch_stage(p, k, l, s, h->G, h->smem, st);
    h->launch_stage(p, ST_LM, 0, s, h->G, h->smem, st);
  }
  XLPK_CUDA(cudaGetLastError());
  advance(h, n_steps, st);
  h->step_base = n_steps;
  return XLPK_OK;
}

xlpk_status xlpk_decode_noalloc(xlpk_handle h, int32_t n_steps, int32_t* tokens_out_dev,
                                const xlpk_decode_io* io, void* stream) {
  xlpk_status rc = check_decode_args(h, n_steps, tokens_out_dev);
  if (rc != XLPK_OK || n_steps == 0) return rc;
  int dev = -1;
  XLPK_CUDA(cudaGetDevice(&dev));
  if (dev != h->device) return XLPK_ERR_INVALID_ARG;
  unsigned char* sc = nullptr;
  rc = noalloc_scratch(dev, &sc);
  if (rc != XLPK_OK) return rc;
  const xlpk_config& c = h->cfg;
  const int B = c.batch, H = c.hidden, d = c.head_dim, F = c.ffn;
  const int qd = c.n_q_heads * d, group = c.n_q_heads / c.n_kv_heads;
  const size_t prow = static_cast<size_t>(B) * c.n_kv_heads * h->G;
  // counters first, so one memset clears everything that must start at zero
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes, 256);
    return o;
  };
  const size_t o_cnt = take(sizeof(unsigned) * h->base.cl.total);
  const size_t cnt_bytes = off;
  const size_t o_x = take(sizeof(float) * B * H);
  const size_t o_q = take(sizeof(float) * B * qd);
  const size_t o_o = take(sizeof(float) * B * qd);
  const int S_moe = h->base.S;
  const size_t o_h = take(sizeof(float) * B * std::max(F, S_moe * c.expert_ffn));
  const size_t o_y = take(sizeof(float) * B * H);
  const size_t o_xacc = take(sizeof(long long) * B * H);
  const size_t o_pml = take(sizeof(float) * prow * group * 2);
  const size_t o_po = take(sizeof(float) * prow * group * d);
  const size_t o_lv = take(sizeof(float) * h->G * B);
  const size_t o_li = take(sizeof(int) * h->G * B);
  const size_t o_rte = take(sizeof(int) * c.n_layers * std::max(S_moe, 1));
  const size_t o_rtw = take(sizeof(float) * c.n_layers * std::max(S_moe, 1));
  if (off > XLPK_NOALLOC_SCRATCH_BYTES) {
    g_cuda_err = "xlpk_decode_noalloc: this handle needs " + std::to_string(off) +
                 " bytes of scratch, more than the " + std::to_string(XLPK_NOALLOC_SCRATCH_BYTES) +
                 "-byte static array";
    return XLPK_ERR_UNSUPPORTED;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Params p = call_params(h, n_steps, tokens_out_dev, io);
  p.step_base = 0;   // fresh counters
  p.cnt = reinterpret_cast<unsigned*>(sc + o_cnt);
  p.x = reinterpret_cast<float*>(sc + o_x);
  p.q = reinterpret_cast<float*>(sc + o_q);
  p.o = reinterpret_cast<float*>(sc + o_o);
  p.h = reinterpret_cast<float*>(sc + o_h);
  p.y = reinterpret_cast<float*>(sc + o_y);
  p.xacc = reinterpret_cast<long long*>(sc + o_xacc);
  p.route_exp = reinterpret_cast<int*>(sc + o_rte);
  p.route_w = reinterpret_cast<float*>(sc + o_rtw);
  p.part_ml = reinterpret_cast<float*>(sc + o_pml);
  p.part_o = reinterpret_cast<float*>(sc + o_po);
  p.lm_val = reinterpret_cast<float*>(sc + o_lv);
  p.lm_idx = reinterpret_cast<int*>(sc + o_li);
  XLPK_CUDA(cudaMemsetAsync(sc, 0, cnt_bytes, st));
  void* args[] = {&p};
  XLPK_CUDA(cudaLaunchCooperativeKernel(h->kern_persistent, dim3(h->G), dim3(kThreads), args,
                                        static_cast<size_t>(h->smem), st));
  for (int b = 0; b < B; ++b) h->pos[b] += n_steps;
  h->last_stream = st;
  return XLPK_OK;
}

xlpk_status xlpk_verify(xlpk_handle h, const int32_t* draft_dev, int32_t n_draft, int32_t* argmax_dev,
                        int32_t* emitted_host, const xlpk_decode_io* io, void* stream) {
  if (!h || !draft_dev || !argmax_dev || !emitted_host || n_draft < 1) return XLPK_ERR_INVALID_ARG;
  if (n_draft != h->cfg.batch - 1 || h->serve_active) return XLPK_ERR_INVALID_ARG;
  if (h->cfg.n_experts > 0) return XLPK_ERR_UNSUPPORTED;
  const int pos = h->pos[0];
  if (pos + n_draft + 1 > h->cfg.max_seq) return XLPK_ERR_KV_FULL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // sequence b > 0 feeds draft b - 1; sequence 0 keeps the pending token
  XLPK_CUDA(cudaMemcpyAsync(h->base.cur_tok + 1, draft_dev, sizeof(int32_t) * n_draft, cudaMemcpyDeviceToDevice, st));
  Params p = call_params(h, 1, argmax_dev, io);
  for (int b = 0; b < h->cfg.batch; ++b) p.pos0[b] = pos + b;
  p.forced = nullptr;
  p.verify = 1;
  p.draft = draft_dev;
  p.accept_out = h->verify_word;
  void* args[] = {&p};
  XLPK_CUDA(cudaLaunchCooperativeKernel(h->kern_persistent, dim3(h->G), dim3(kThreads), args,
                                        static_cast<size_t>(h->smem), st));
  h->last_stream = st;
  XLPK_CUDA(cudaMemcpyAsync(emitted_host, h->verify_word, sizeof(int32_t), cudaMemcpyDeviceToHost, st));
  const xlpk_status rc = xlpk_get_status(h);   // synchronises the stream
  if (rc != XLPK_OK) return rc;
  const int n = *emitted_host;
  for (int b = 0; b < h->cfg.batch; ++b) h->pos[b] = pos + n;
  h->step_base += 1;
  return XLPK_OK;
}

xlpk_status xlpk_debug_logits(xlpk_handle h, float* logits_dev, float* hidden_dev) {
  if (!h) return XLPK_ERR_INVALID_ARG;
  if ((logits_dev && !aligned16(logits_dev)) || (hidden_dev && !aligned16(hidden_dev))) return XLPK_ERR_INVALID_ARG;
  h->dbg_logits = logits_dev;
  h->dbg_hidden = hidden_dev;
  return XLPK_OK;
}

xlpk_status xlpk_generate(xlpk_handle h, const int32_t* tokens_host, const int32_t* seq_lens_host,
                          int32_t n_steps, int32_t* tokens_out_host, void* stream) {
  if (!h || !tokens_out_host) return XLPK_ERR_INVALID_ARG;
  if (n_steps < 0 || n_steps > h->cfg.max_seq) return XLPK_ERR_INVALID_ARG;
  xlpk_status rc = xlpk_set_state(h, tokens_host, seq_lens_host, stream);
  if (rc != XLPK_OK) return rc;
  rc = xlpk_decode(h, n_steps, h->tok_scratch, nullptr, stream);
  if (rc != XLPK_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  XLPK_CUDA(cudaMemcpyAsync(tokens_out_host, h->tok_scratch,
                            sizeof(int32_t) * static_cast<size_t>(n_steps) * h->cfg.batch,
                            cudaMemcpyDeviceToHost, st));
  return xlpk_get_status(h);
}

xlpk_status xlpk_get_status(xlpk_handle h) {
  if (!h) return XLPK_ERR_INVALID_ARG;
  XLPK_CUDA(cudaStreamSynchronize(h->last_stream));
  int st[4] = {0, 0, 0, 0};
  XLPK_CUDA(cudaMemcpy(st, h->base.status, sizeof(st), cudaMemcpyDeviceToHost));
  if (st[0] == 0) return XLPK_OK;
  // reset the device-side ordering state so the handle is usable again
  XLPK_CUDA(cudaMemset(h->base.cnt, 0, sizeof(unsigned) * h->base.cl.total));
  XLPK_CUDA(cudaMemset(h->base.status, 0, sizeof(int) * 4));
  XLPK_CUDA(cudaMemset(h->base.abort_flag, 0, sizeof(int)));
  XLPK_CUDA(cudaDeviceSynchronize());
  h->step_base = 0;
  char buf[160];
  if (st[0] == XLPK_ERR_INVALID_ARG)
    std::snprintf(buf, sizeof(buf), "a KV page-table entry outside the pool: stage %d layer %d step %d cta %d",
                  st[1] & 0xff, (st[1] >> 8) & 0xff, (st[1] >> 16) & 0x7fff, st[2]);
  else
    std::snprintf(buf, sizeof(buf), "device wait failed: stage %d layer %d step %d cta %d", st[1] & 0xff,
                  (st[1] >> 8) & 0xff, (st[1] >> 16) & 0x7fff, st[2]);
  g_cuda_err = buf;
  return static_cast<xlpk_status>(st[0]);
}

xlpk_status xlpk_get_info(xlpk_handle h, xlpk_info* out) {
  if (!h || !out) return XLPK_ERR_INVALID_ARG;
  out->n_ctas = h->G;
  out->threads_per_cta = kThreads;
  out->smem_bytes = h->smem;
  out->ring_slots = h->nslot;
  out->slot_bytes = kSlotBytes;
  out->kernels_per_step_unfused = h->cfg.n_layers * (h->ffn_fused ? ST_LAYER - 1 : ST_LAYER) + 1;
  out->packed_weight_bytes = static_cast<int64_t>(h->packed_bytes);
  out->workspace_bytes = static_cast<int64_t>(h->ws_bytes);
  out->weight_bytes_per_step = h->weight_bytes_per_step;
  return XLPK_OK;
}

const char* xlpk_status_string(int32_t s) {
  switch (s) {
    case XLPK_OK: return "XLPK_OK";
    case XLPK_ERR_INVALID_ARG: return "XLPK_ERR_INVALID_ARG";
    case XLPK_ERR_UNSUPPORTED: return "XLPK_ERR_UNSUPPORTED";
    case XLPK_ERR_CUDA: return "XLPK_ERR_CUDA";
    case XLPK_ERR_OOM: return "XLPK_ERR_OOM";
    case XLPK_ERR_KV_FULL: return "XLPK_ERR_KV_FULL";
    case XLPK_ERR_TIMEOUT: return "XLPK_ERR_TIMEOUT";
    case XLPK_ERR_ABORTED: return "XLPK_ERR_ABORTED";
    default: return "XLPK_ERR_UNKNOWN";
  }
}

const char* xlpk_last_cuda_error(void) { return g_cuda_err.c_str(); }

}  // extern "C"

// ---- tensor-core tile entry point: separate from the persistent decode (the
// decode's kernels and planning above do not depend on anything below)

#include "tc_tile.cuh"

// Error word of xlpk_tc_gemm_tile (one call at a time per process).
static __device__ int g_tc_err;

extern "C" xlpk_status xlpk_tc_gemm_tile(const void* w_dev, int32_t n, int32_t k, const float* x_dev,
                                         float* y_dev, void* stream) {
  if (!w_dev || !x_dev || !y_dev) return XLPK_ERR_INVALID_ARG;
  if (n < kTcRows || k < kTcKBox || k > kTcMaxK || k % kTcKBox) return XLPK_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(w_dev) | reinterpret_cast<uintptr_t>(x_dev) |
       reinterpret_cast<uintptr_t>(y_dev)) & 15u)
    return XLPK_ERR_INVALID_ARG;
  int dev = -1;
  XLPK_CUDA(cudaGetDevice(&dev));
  int major = 0;
  XLPK_CUDA(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev));
  if (major != 10) {
    g_cuda_err = "device is not sm_100";
    return XLPK_ERR_UNSUPPORTED;
  }
  // the weight matrix as a 2-D [n][k] bf16 array read in [128 rows][64 columns]
  // boxes with 128-byte swizzle: the layout of the MMA's A operand
  CUtensorMap map;
  xlpk_status rc = encode_kv_map(&map, const_cast<void*>(w_dev), static_cast<unsigned long long>(n), k, kTcRows);
  if (rc != XLPK_OK) return rc;
  const int smem = tc_smem_bytes(k);
  XLPK_CUDA(cudaFuncSetAttribute(tc_gemm_tile_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
  int* err = nullptr;
  XLPK_CUDA(cudaGetSymbolAddress(reinterpret_cast<void**>(&err), g_tc_err));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  XLPK_CUDA(cudaMemsetAsync(err, 0, sizeof(int), st));
  tc_gemm_tile_kernel<<<(n + kTcRows - 1) / kTcRows, kTcThreads, smem, st>>>(map, n, k, x_dev, y_dev, err,
                                                                             200000000LL);
  XLPK_CUDA(cudaGetLastError());
  XLPK_CUDA(cudaStreamSynchronize(st));
  int e = 0;
  XLPK_CUDA(cudaMemcpy(&e, err, sizeof(int), cudaMemcpyDeviceToHost));
  if (e != 0) {
    g_cuda_err = "xlpk_tc_gemm_tile: a device wait ran out";
    return static_cast<xlpk_status>(e);
  }
  return XLPK_OK;
}
