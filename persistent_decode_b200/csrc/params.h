// Shared host/device description of one decode launch.
//
// The host planner (xlpk.cu) fills these at xlpk_create time; the kernels in
// engine.cuh read them.  Everything a CTA needs to find its tiles is here or
// derivable from (CTA index, grid size, step), so no per-task table has to be
// fetched at run time: the "task list" of a CTA is the static partition of
// every stage's rows (or attention chunks) by CTA index.
#pragma once
#include <cuda.h>   // CUtensorMap (type only; the library does not link libcuda)
#include <stdint.h>

namespace xlpk {

constexpr int kConsumerWarps = 8;
constexpr int kConsumerThreads = kConsumerWarps * 32;
constexpr int kThreads = kConsumerThreads + 32;      // + one producer warp
constexpr int kTileBytes = 32768;                     // data of one tile: weights, or a K and a V chunk
constexpr int kSlotBytes = kTileBytes + 1024;         // ring slot stride: + FP8 tiles' per-row block scales
constexpr int kMaxSlots = 8;
// Ring depth and L2-prefetch distance of the CUDA-core decode (batch <= 4,
// dense or MoE).  There the short stages (QKV, attention, O-projection) wait on
// their input copy, and every weight copy already queued on the SM (the ring's
// slots for the next stage) and every prefetch in flight delay it: a ring of 4
// slots and a 128 KB prefetch distance decode 0.5-9 % faster than 5-8 slots
// and 256 KB.  (The batch-8 tensor-core decode keeps as many slots as fit.)
constexpr int kShallowSlots = 4;
constexpr long long kShallowPrefetchBytes = 128 * 1024;
constexpr long long kPrefetchBytes = 256 * 1024;
constexpr int kMaxBatch = 8;
constexpr int kMaxGroup = 4;                          // query heads per kv head
constexpr int kPairsPerTile = kConsumerWarps;         // one row pair per consumer warp
constexpr int kMiscSmem = 4096;                       // barriers, flags, reduction scratch
constexpr int kMaxExperts = 256;                      // routed experts per MoE layer
constexpr int kMaxMoeSlots = 16;                      // shared + selected experts per token
constexpr int kMaxCtas = 160;                        // persistent grid limit (one CTA per SM; B200 has 148)
constexpr int kTraceSlots = 16;                       // u64 stamps per (step, stage, CTA) in a trace
constexpr int kMaxWinGroups = 4;                      // K-windowed down projection: row-pair groups per CTA

// Stages of one layer, in dependency order, then the LM head.
enum StageKind : int {
  ST_QKV = 0,     // RMSNorm(x) -> [q;k;v] GEMV, RoPE, KV append
  ST_ATTN = 1,    // flash-decoding split over the sequence + last-arriver combine
  ST_OPROJ = 2,   // x += Wo o   (layer 0: x = E[tok] + Wo o)
  ST_GATEUP = 3,  // h = silu(Wg xn) * (Wu xn)
  ST_DOWN = 4,    // x += Wd h
  ST_LAYER = 5,   // stages per layer
  ST_LM = 5       // logits = Wlm RMSNorm(x), argmax, next token
};

// Counter slots (unsigned, monotonic unless noted).
//   cnt[l*ST_LAYER + kind]   arrivals of stage `kind` of layer l: G per step,
//                            except ST_ATTN which counts finished (b, kv-head)
//                            combines: B*n_kv per step.
//   cnt[lm_arrive]           G per step
//   cnt[step_done]           1 per step
//   cnt[attn_arrive + ...]   per (layer, b, kv head) chunk arrivals, reset to 0
//                            by the CTA that completes the head.
struct CounterLayout {
  int lm_arrive;
  int step_done;
  int attn_arrive;
  int total;
};

// A packed GEMV operand: logical rows are grouped in pairs; the pairs are
// split evenly over the CTAs; a CTA's pairs are cut into groups of up to 8
// (one pair per consumer warp) and each group into k-chunks of KC columns.
// Tile (group, chunk) holds [2*gp rows][KC cols] contiguously, and the tiles
// of a CTA follow each other, so the CTA's whole span is one contiguous range
// streamed front to back.
//
// FP8 (e4m3) matrices: each tile's [2*gp rows][KC codes] is followed by the
// rows' block scales [2*gp rows][KC/128] fp32 (the scale of the row's 128x128
// block for each 128 columns of the chunk), so a tile still arrives as one
// bulk copy; a packed row then takes K + K/32 bytes.
struct Mat {
  const uint8_t* packed;
  const float2* gsc;     // NVFP4: per row pair, the two rows' matrix scales; else null
  int N;                 // logical rows (even)
  int K;                 // columns
  int KC;                // k-chunk (divides K)
  int fp8;               // 1: e4m3 codes + in-tile fp32 scales per 128x128 block
  int fp4;               // 1: NVFP4 e2m1 codes + in-tile e4m3 scales per 16 columns (and gsc)
};

// Bytes of one packed row over `k` columns (codes or bf16 values, plus the
// in-tile block scales: FP8 one fp32 per 128 columns, NVFP4 one byte per 16).
__host__ __device__ __forceinline__ int packed_row_bytes(const Mat& m, int k) {
  return m.fp4 ? k / 2 + k / 16 : m.fp8 ? k + k / 32 : 2 * k;
}

// ------------------------------------------------------------------ batch-8 tensor-core tiles
// With Params::tc (batch 8, dense layers) every projection runs on tcgen05
// MMAs.  A CTA owns an even share of the matrix's 8-row units; its rows form
// M-tiles of up to 128 rows.  Weights are packed per CTA span in (K window,
// M-tile, tile) order; a tile is nb boxes of [rv rows][128 bytes] (64 bf16 or
// 128 e4m3 columns), each box in the canonical K-major 128-byte-swizzle layout
// (row r's 16-byte unit q at r*128 + ((q ^ (r % 8)) * 16)), followed for FP8 by
// the rows' block scales [nb][rv] fp32.  A plain bulk copy of a tile into a
// 1024-byte-aligned ring slot therefore lands as nb ready MMA operands.
__host__ __device__ inline int tc_box_cols(int fp8) { return fp8 ? 128 : 64; }
// Boxes per tile for M-tiles of rv rows: the largest power of two <= 16 whose
// tile fits (bf16: 32 KB; FP8 codes: 16 KB, so that their in-place bf16
// expansion fits the slot), whose last bf16 box still leaves the 128 rows an
// M = 128 MMA reads inside the slot, and which divides `kbox`, the boxes per K
// window.
__host__ __device__ inline int tc_nb(int rv, int kbox, int fp8) {
  const int cap = fp8 ? 16384 : 32768;
  int nb = 16;
  while (nb > 1 && (nb * rv * 128 > cap || ((fp8 ? 2 : 1) * nb - 1) * rv * 128 + 128 * 128 > kSlotBytes ||
                    kbox % nb))
    nb >>= 1;
  return nb;
}
__host__ __device__ inline int tc_tile_bytes(int rv, int nb, int fp8) { return nb * rv * 128 + (fp8 ? nb * rv * 4 : 0); }
// Packed bytes of one row over `cols` columns (codes or values + FP8 scales).
__host__ __device__ inline long long tc_row_bytes(long long cols, int fp8) { return fp8 ? cols + cols / 32 : 2 * cols; }
__host__ __device__ inline int tc_gcd(int a, int b) {
  while (b) {
    const int t = a % b;
    a = b;
    b = t;
  }
  return a;
}
// K window of a tensor-core projection: Params::tc_win columns when K is
// larger (the activation region holds one window of the B operand), else 0
// (the whole K at once).
__host__ __device__ inline int tc_window(int tc_win, int K) { return tc_win > 0 && K > tc_win ? tc_win : 0; }
// Boxes per window common to every window of a K x (window) split.
__host__ __device__ inline int tc_kbox(int K, int win, int fp8) {
  const int bc = tc_box_cols(fp8);
  return win > 0 ? tc_gcd(K / bc, win / bc) : K / bc;
}

struct LayerParams {
  Mat qkv;     // rows: q heads (RoPE pairs interleaved), k heads (interleaved), v heads
  Mat o;
  Mat gu;      // rows: gate_j, up_j interleaved (dense layers)
  Mat down;    // dense layers
  const float* attn_norm;
  const float* ffn_norm;
  // MoE layers.  Experts are numbered 0..E-1 (routed) then E..E+S_sh-1
  // (shared).  The router and every expert's gate/up are packed as one
  // block streamed whole (groups of 8 row pairs in order, not split over the
  // CTAs); every expert's down projection is packed like a dense matrix
  // (rows split over the CTAs).  egu / edown describe expert 0; expert e's
  // block starts e * egu_stride (edown_stride) bytes further.
  // Dense layers with the fused FFN stage: W_down transposed, bf16 [F][H]
  // row-major; a CTA streams the rows (= W_down columns) matching its own
  // gate/up pairs.
  Mat downT;
  Mat router;
  Mat egu;
  Mat edown;
  long long egu_stride;
  long long edown_stride;
};

struct Params {
  // shape
  int L, H, nq, nkv, d, F, V, B, max_seq;
  int E, topk, nsh, S, Fe;  // MoE: routed experts, selected per token, shared, slots (nsh + topk), expert width
  int group;            // nq / nkv
  int esz;              // weight bytes per element (2 bf16, 1 fp8)
  float eps;
  float qk_scale_log2;  // log2(e) / sqrt(d)
  int G;                // CTAs
  int nslot;            // ring slots in use
  int act_bytes;        // activation / scratch region
  int side_bytes;       // epilogue side region (after the activation region)
  int side_rope;        //   byte offset of the RoPE rows [B][d/2] float2
  int side_resid;       //   byte offset of the residual slice [B][2 planes][nvr] float4
  int side_embed;       //   byte offset of the embedding slice [B][evb bytes]
  int nvr;              //   float4 vectors per (sequence, plane) of the residual slice
  int rows_side;        //   fused-FFN layers: int64 rows per sequence of the accumulator slice
  int evb;              //   bytes per sequence of the embedding slice
  int attn_pos_per_tile;
  long long spin_limit_ns;
  unsigned wait_hint_ns;  // suspend-time hint of mbarrier waits (0: plain polling)
  long long l2_prefetch_bytes;  // how far the producer's L2-prefetch cursor runs ahead
  CounterLayout cl;

  // weights
  const uint16_t* embed;        // bf16 [V][H]
  const float* final_norm;
  Mat lm;
  const LayerParams* layers;    // device array [L]

  // KV cache (caller-owned), bf16 [L][B][nkv][max_seq][d], or paged: pools
  // [L][n_pages][nkv][P][d] with P = attn_pos_per_tile; the tensor maps view
  // each as a 2-D [rows][d] array read in 64-column boxes of P rows with
  // 128-byte swizzle
  CUtensorMap tmap_k;
  CUtensorMap tmap_v;
  uint16_t* kc;          // bf16 cache (null for an e4m3 cache)
  uint16_t* vc;
  uint8_t* kc8;          // e4m3 cache: codes (null for a bf16 cache)
  uint8_t* vc8;
  int kv_fp8;            // 1: the cache holds e4m3 codes; entry = code * k_scale / v_scale
  float k_inv, v_inv;    // 1 / k_scale, 1 / v_scale (powers of two)
  float k_scale, v_scale;
  const int32_t* page_table;   // paged cache: [B][pages_per_seq] pool page of each chunk; null: contiguous
  int pages_per_seq;
  int n_pages;
  const float2* rope;           // [max_seq][d/2] (cos, sin)

  // workspace
  float* x;          // [B][H] residual stream (two-plane fp32; layers without the fused FFN)
  long long* xacc;   // fused FFN: [B][H] residual stream, 64-bit fixed point with 32 fractional
                     // bits, into which the down projection's split-K partials are added
  float* q;          // [B][nq*d] rotated queries
  float* o;          // [B][nq*d] attention output
  float* h;          // [B][F] SwiGLU output (MoE: [B][S*Fe], slot-major, gate-weighted)
  float* y;          // fused FFN: [B][H] residual after attention (the FFN's RMSNorm input);
                     // xacc then accumulates the down projection's partial sums
  int ffn_fused;     // 1: gate/up and down run as one stage with a split-K down projection
  int resid_fixed;   // fused FFN: 1 = residual in the fixed-point accumulator xacc (bit-reproducible
                     // integer split-K adds), 0 = two-plane fp32 x with float atomics
  int jt;            // fused FFN: W_down columns per tile
  int tc;            // 1: batch-8 projections on tcgen05 MMAs (tensor-core packing and stages)
  int tc_cols;       //   tensor-memory columns each CTA allocates (16 per M-tile of its largest stage)
  int tc_win;        //   K window of the tensor-core projections (tc_window), 0: whole K
  int down_win;      // K-windowed down projection: W_down columns per activation window (0: whole K);
                     // the CTA's down tiles are packed window by window, groups inside a window
  int side_hloc;     // fused FFN: byte offset of the CTA's h slice [B][hloc] in the side region
  int hloc;          //   floats per sequence of that slice (max gate/up pairs per CTA)
  int* route_exp;    // MoE: [L][S] expert of each slot (written by CTA 0)
  float* route_w;    // MoE: [L][S] weight of each slot
  float* part_ml;    // [B][nkv][G][group][2] per contributing CTA: (max in log2 units, sum)
  float* part_o;     // [B][nkv][G][group][d] unnormalised attention output
  float* lm_val;     // [G][B]
  int* lm_idx;       // [G][B]
  unsigned* cnt;
  int* cur_tok;      // [B] pending input token
  int* status;       // [0] error code, [1] where
  int* abort_flag;

  // per call
  int n_steps;
  int step_base;     // global index of this call's first step
  int pos0[kMaxBatch];
  int32_t* tokens_out;
  const int32_t* forced;
  float* logits_out;
  float* hidden_out;
  int logits_overwrite;        // 1: every step writes logits_out[0..B) (parity mode), else step s at [s]
  int hidden_overwrite;        // the same for hidden_out
  int32_t* experts_out;        // MoE: [n_steps][L][B][topk] selected experts (may be null)
  unsigned long long* trace;   // optional stage timestamps
  int fault_drop_stage;        // failure-detection tests: CTA 0 withholds its release of this
                               // stage index at the call's first step (-1: never)

  // Speculative verify (one step): sequence b is the pending token (b = 0) or
  // draft b - 1 fed at position pos0[b] = pos0[0] + b; every sequence reads the
  // same pages, so attention needs this step's KV rows of the sequences before
  // it (the producer waits for this step's QKV stage, not the previous one's).
  // The LM head's last arriver accepts the longest prefix of drafts equal to the
  // argmaxes and writes the number of tokens emitted (accepted + 1) to accept_out.
  int verify;
  const int32_t* draft;        // [B - 1] draft tokens
  int32_t* accept_out;         // [1]

  // Device-resident request loop (serve mode): launch step s runs once the
  // host has asked for more than serve_step0 + s steps of the session.  CTA 0's
  // first consumer thread polls the host-mapped request word and forwards it to
  // serve_req_dev, which every other CTA polls; when no request comes for
  // serve_idle_ns (or the host asks to leave while idle), CTA 0 names the step
  // at which every CTA stops (serve_stop_dev) and the launch ends.
  int serve;
  int serve_step0;                  // session index of this launch's step 0
  const unsigned* serve_req_host;   // host-mapped: steps requested in the session
  const int* serve_exit_host;       // host-mapped: 1 = leave when idle
  unsigned* serve_done_host;        // host-mapped: steps completed in the session
  int32_t* serve_tokens_host;       // host-mapped ring [serve_cap][B]: token of session step t at t % cap
  int serve_cap;
  unsigned* serve_req_dev;          // workspace: the request count as CTA 0 forwarded it
  int* serve_stop_dev;              // workspace: launch step at which every CTA leaves (-1: none yet)
  long long serve_idle_ns;
};

}  // namespace xlpk
