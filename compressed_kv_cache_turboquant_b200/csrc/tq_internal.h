// Internal declarations shared by the host API and the kernels.
#pragma once

#include <nvtx3/nvToolsExt.h>
#include <cstddef>
#include <cstdint>

#include "tq.h"

namespace tqi {
// An NVTX range named after the C entry point for the duration of the call
// (host side: argument checks and launches), so a profiler's timeline shows
// the library's calls; free when no tool is attached.
struct TraceRange {
  explicit TraceRange(const char* name) { nvtxRangePushA(name); }
  ~TraceRange() { nvtxRangePop(); }
  TraceRange(const TraceRange&) = delete;
  TraceRange& operator=(const TraceRange&) = delete;
};
}  // namespace tqi
#define TQ_TRACE(name) ::tqi::TraceRange tq_trace_range_(name)

namespace tqi {

// Thread-local error text behind tq_last_error(); returns `code` for chaining.
int set_error(int code, const char* fmt, ...);
int clear_error();

// Let a kernel use a dynamic shared-memory window of `bytes` on the current
// device: its limit is raised to the device's opt-in maximum once per
// (kernel, device) -- the setting belongs to the device current when it is
// made.  Safe to call from several host threads.  Returns a cudaError_t.
int ensure_dyn_smem(const void* kernel, int bytes);

constexpr int kMaxMseBits = 4;

// Device-resident constants of one quantizer instance (one cudaMalloc block).
struct DevConsts {
  float* Pi = nullptr;          // [d][d] row-major, y = Pi x
  float* PiT = nullptr;         // [d][d] row-major transpose of Pi
  float* S = nullptr;           // [d][d] QJL projection (prod), for the query side S q
  float* TT = nullptr;          // [d][d] transpose of T = S Pi^T (prod): [i][j] = T[j][i]
  float* centroids = nullptr;   // [2^bm]
  float* thresholds = nullptr;  // [2^bm - 1]
  // tensor-core operands: rotation / projection split into bf16 pieces,
  // pre-arranged in the shared-memory layout the MMA kernels consume
  uint16_t* Pi_bf16 = nullptr;  // [pieces][d*d]
  uint16_t* T_bf16 = nullptr;   // [pieces][d*d]
  // decode tables
  uint32_t* lut_f16 = nullptr;  // packed fp16 centroid byte tables
  // rotation split into 3 bf16 pieces (hi, mid, lo) laid out as the tensor-core
  // kernels hold them in shared memory: [piece][K slab of 64][row j][128 B,
  // 16-byte chunks XOR-swizzled by row % 8]; only for d in {64, 128}
  uint8_t* pi_tc = nullptr;
  int* status = nullptr;        // device status word (bounded waits that expired)
  // Pi^T in two fp16 pieces (hi, lo * 2^11), same swizzled K-major layout, and
  // the centroid table as fp16 pieces (hi | lo * 2^11 << 16), for dequant
  uint8_t* pit_f16 = nullptr;
  uint32_t* lut_dq = nullptr;
  // fp16 byte tables for register decoding (byte-permute lookups):
  // ktab (3-bit codebooks): lo bytes of c0..3, c4..7, hi bytes of c0..3, c4..7
  // vtab (4-bit symmetric codebooks): the same for the upper half c8..c15
  uint32_t* ktab = nullptr;
  uint32_t* vtab = nullptr;
  // general-d quantizer operands, fp16 row-major, d_pad = d rounded up to 128,
  // zero padded: gen_pi = [hi; lo * 2^11] of Pi as [2 d_pad][d_pad] (row = output
  // coordinate, column = input coordinate); gen_st (prod) = [hi; lo * 2^11] of
  // [S | T] as [2 d_pad][2 d_pad]
  uint16_t* gen_pi = nullptr;
  uint16_t* gen_st = nullptr;
  // fused quantizer operands (d <= 256): fp16 pieces (hi, and the remainder
  // itself as lo) of kFusedPieceScale * Pi and (prod) of kFusedPieceScale * T,
  // each [2][n16][k64] (row = output coordinate, column = input coordinate,
  // n16 = d rounded up to 16, k64 = d rounded up to 64, zero padded)
  uint16_t* fz_pi = nullptr;
  uint16_t* fz_t = nullptr;
};

// scale of the fused quantizer's constant pieces: keeps their fp16 remainders normal
constexpr float kFusedPieceScale = 1024.f;

}  // namespace tqi

struct tq_ctx {
  int d = 0, b = 0, variant = 0, bm = 0;  // bm: mse bits (b for MSE, b-1 for PROD)
  int device = 0;
  int sm_count = 0;
  void* block = nullptr;  // the single device allocation
  size_t block_bytes = 0;
  tqi::DevConsts dev;
  // host copies (float64) kept for diagnostics
  double host_centroids[16] = {0};
  double host_thresholds[15] = {0};
  // fp16 codebook for the tensor-core scorer: sc_tab[k] = fp16(alpha c[k]) with
  // one fp32 scale alpha in [1, 2) chosen so the scaled centroids are as close
  // to fp16 values as possible; products are divided by alpha in fp32
  uint16_t sc_tab[16] = {0};
  float sc_inv_alpha = 1.f;
  int gen_d_pad = 0;
  uint32_t dyn_base = 0xFFFFFFFFu;  // shared address of a kernel's dynamic window (probed at creation)
  // Diagnostics read from the environment at creation (normally off):
  //   TQ_DEBUG_STALL_MS=m   the decode kernel's consumer warps first wait, m ms
  //                         at most, on a barrier that nothing completes, and
  //                         every other wait of that kernel gives up after m ms:
  //                         the timeout path runs and reports TQ_STATUS_TIMEOUT
  //   TQ_DEBUG_DYN_BASE=a   record `a` as the measured shared-window address:
  //                         the decode and logits kernels built for the usual
  //                         address run and find the window elsewhere
  //                         (TQ_STATUS_LAYOUT)
  uint64_t debug_stall_ns = 0;
  int fz_n16 = 0, fz_k64 = 0;  // fused quantizer tile shape (0: not available)
  // TQ_FUSED_REGISTER_LOADS=1 at creation: contiguous inputs take the fused
  // quantizer whose producer threads load x themselves (the one a channel
  // gather always takes) instead of the TMA-staged one
  bool fused_register_loads = false;
  // PolarQuant (variant TQ_POLAR): level-1 bits, bits of levels >= 2, tan^2 of
  // the thresholds of levels 2..7 and the cos / sin of every level's centroids
  int polar_b1 = 0, polar_bh = 0;
  float polar_tan2[8][3] = {};
  float* polar_cs = nullptr;  // device [2][8 levels][16]: cos, sin of centroid k of level l (level 1 at l = 1)
  bool debug_fixed_tables = false;  // TQ_DEBUG_DYN_BASE given: take the fixed-address kernels anyway
  // TQ_TCGEN05_ATTN=1 at creation: dense decode and split-cache logits take
  // the tcgen05 kernels instead of the mma.sync ones (both are covered by the
  // parity tests; the mma.sync kernels are faster today)
  bool tc_attn = false;
  // 3-bit codebook as fp16 byte tables (register decoding): lo bytes of c0-3,
  // c4-7, hi bytes of c0-3, c4-7 (zero unless b = 3 mse bits)
  uint32_t host_ktab[4] = {0, 0, 0, 0};
  double sc_rel_err = 0.0;  // max |fp16(alpha c) / alpha - c| / |c|
};

namespace tqi {

// A paged K/V cache (page > 0): token t of (batch, kv-head) bh is row
// block_table[bh * max_pages + t / page] * page + t % page of every array;
// page == 0 is the dense layout (row bh * kv_stride + t).  rn16: the residual
// norms are stored as fp16.
struct PagedCache {
  const int32_t* block_table = nullptr;
  int max_pages = 0;
  int page = 0;
  int rn16 = 0;
};

// number of context splits tq_attn_decode uses for a (B, Hq, T) problem
int probe_dyn_smem_base(uint32_t* scratch, uint32_t* base);
int decode_splits(int B, int Hq, int64_t T, int sm_count);

// ---- launchers (kernels_*.cu); all return cudaError_t as int ----
bool quant_tc_supported(const tq_ctx* h, int dtype);
bool dequant_tc_supported(const tq_ctx* h);
int launch_dequant_tc(const tq_ctx* h, const uint32_t* codes, const float* norms, int64_t N, void* out,
                      int out_dtype, void* stream);
int launch_quant_mse_tc(const tq_ctx* h, const void* x, int64_t N, int64_t x_stride, uint32_t* codes,
                        float* norms, int64_t out_stride, void* stream);
int launch_quant_simple(const tq_ctx* h, const void* x, int dtype, int64_t N, int64_t x_stride,
                        uint32_t* codes, uint32_t* signs, float* norms, float* rnorms,
                        int64_t out_stride, void* stream, const int32_t* channels = nullptr);
// one launch for up to two channel groups of N vectors (d <= 256 each; N < 65536)
int launch_quant_small(const tq_ctx* const* h, int ngroups, const void* x, int dtype, int64_t N, int64_t x_stride,
                       const int32_t* channels, uint32_t* const* codes, uint32_t* const* signs, float* const* norms,
                       float* const* rnorms, int64_t out_stride, void* stream);
int launch_query_prep_gather(const tq_ctx* h, const void* q, int q_dtype, int64_t nq, int dq,
                             const int32_t* channels, float* qrot, float* qproj, void* stream);
bool quant_gen_supported(const tq_ctx* h);
// n_i = ||x_i|| in float64 -> norms[out row of i] (channels / slots as for the fused quantizer)
int launch_gen_norms(const tq_ctx* h, const void* x, int dtype, int64_t N, int64_t x_stride, float* norms,
                     int64_t out_stride, void* stream, const int32_t* channels = nullptr,
                     const int64_t* slots = nullptr);
bool quant_fused_supported(const tq_ctx* h);
// the fused quantizer with the input staged by TMA and the residual in tensor
// memory (rows of x start 16-byte aligned; no channel gather)
int launch_quant_fused2(const tq_ctx* h, const void* x, int dtype, int64_t N, int64_t x_stride, uint32_t* codes,
                        uint32_t* signs, float* norms, void* rnorms, int64_t out_stride, void* stream,
                        const int64_t* slots, int rn_f16);
// d <= 256: norms, then one persistent tensor-core kernel for codes (and QJL bits, ||r||).
// channels: optional gather of each row's d channels; slots: optional output row per
// vector (else i * out_stride); rn_f16: rnorms is __half storage
int launch_quant_fused(const tq_ctx* h, const void* x, int dtype, int64_t N, int64_t x_stride, uint32_t* codes,
                       uint32_t* signs, float* norms, void* rnorms, int64_t out_stride, void* stream,
                       const int32_t* channels = nullptr, const int64_t* slots = nullptr, int rn_f16 = 0);
bool quant_gen_needs_workspace(const tq_ctx* h);
size_t quant_gen_workspace_rows_bytes(const tq_ctx* h);
int launch_quant_gen(const tq_ctx* h, const void* x, int dtype, int64_t N, int64_t x_stride, uint32_t* codes,
                     uint32_t* signs, float* norms, float* rnorms, int64_t out_stride, void* workspace,
                     size_t ws_bytes, void* stream);
bool scores_tc_supported(const tq_ctx* h, int topk);
size_t scores_tc_workspace(const tq_ctx* h, int64_t nq, int64_t N, int topk);
int launch_scores_tc(const tq_ctx* h, const float* q, int64_t nq, const uint32_t* codes, const uint32_t* signs,
                     const float* norms, const float* rnorms, int64_t N, float* scores, int topk, int32_t* top_idx,
                     float* top_val, void* workspace, void* stream);
bool logits_supported(const tq_ctx* const* hk, int ngroups);
bool logits_mma_supported(const tq_ctx* const* hk, int ngroups, int64_t kv_stride);
size_t logits_mma_workspace(int64_t nq);
int launch_logits_mma(const tq_ctx* const* hk, const float* const* qrot, const float* const* qproj, int B, int Hq,
                      int Hkv, int64_t T, int64_t kv_stride, const uint32_t* const* kcodes,
                      const uint32_t* const* ksigns, const float* const* knorms, const float* const* krnorms,
                      float scale, float* logits, void* workspace, void* stream);
int launch_logits(const tq_ctx* const* hk, int ngroups, const float* const* qrot, const float* const* qproj, int B,
                  int Hq, int Hkv, int64_t T, int64_t kv_stride, const uint32_t* const* kcodes,
                  const uint32_t* const* ksigns, const float* const* knorms, const float* const* krnorms,
                  float scale, float* logits, void* stream);
int launch_dequant_simple(const tq_ctx* h, const uint32_t* codes, const float* norms, int64_t N,
                          void* out, int out_dtype, void* stream);
int launch_query_prep(const tq_ctx* h, const float* q, int q_dtype, int64_t nq, float* qrot,
                      float* qproj, void* stream);
int launch_scores_simple(const tq_ctx* h, const float* qrot, const float* qproj, int64_t nq,
                         const uint32_t* codes, const uint32_t* signs, const float* norms,
                         const float* rnorms, int64_t N, float* scores, void* stream);
int launch_topk_simple(const float* scores, int64_t nq, int64_t N, int k, int32_t* top_idx,
                       float* top_val, void* stream);
// merge of decode partials: split s of row bh at partials + bh * row_stride + s * split_stride;
// partial_out writes the merged (acc, m, l) record [BH][d + 2] instead of the rotated output
int launch_decode_merge(const float* partials, int64_t BH, int splits, const tq_ctx* hv, float* out,
                        void* stream, int64_t split_stride, int64_t row_stride, int partial_out = 0);
bool decode_mma_supported(const tq_ctx* hk, const tq_ctx* hv, int Hq, int Hkv, int64_t kv_stride);
int decode_mma_grid(int B, int Hkv, int64_t T, int sm_count);
int decode_mma_max_seg(int B, int Hkv, int64_t T, int sm_count);
int launch_qfrag(const float* qrot, const float* qproj, int64_t nq, void* qfrag, float* qscale, void* stream);
// combine the per-CTA softmax records of a persistent decode kernel (block
// partition of `total` blocks, nblk per (batch, kv-head), max_seg records per
// CTA and head) and rotate back once
int launch_decode_merge_records(const float* partials, int64_t G, int max_seg, int64_t nblk, int64_t total, int B,
                                int Hq, int Hkv, const tq_ctx* hv, float* out, int partial_out, void* stream);
// split-cache logits on tcgen05
bool logits_tc_supported(const tq_ctx* const* hk, int ngroups, int64_t kv_stride);
size_t logits_tc_workspace(int B, int Hkv);
int launch_logits_tc(const tq_ctx* const* hk, const float* const* qrot, const float* const* qproj, int B, int Hq,
                     int Hkv, int64_t T, int64_t kv_stride, const uint32_t* const* kcodes,
                     const uint32_t* const* ksigns, const float* const* knorms, const float* const* krnorms,
                     float scale, float* logits, void* workspace, void* stream);
// decode attention on tcgen05 (dense cache)
bool decode_tc_supported(const tq_ctx* hk, const tq_ctx* hv, int Hq, int Hkv, int64_t kv_stride, int rn16);
int decode_tc_grid(int B, int Hkv, int64_t T, int sm_count);
int decode_tc_max_seg(int B, int Hkv, int64_t T, int sm_count);
size_t decode_tc_qtile_bytes(int B, int Hkv);
int launch_decode_tc(const tq_ctx* hk, const tq_ctx* hv, const float* qrot, const float* qproj, uint8_t* qtiles,
                     float* qscale, int B, int Hq, int Hkv, int64_t T, int64_t kv_stride, const uint32_t* kcodes,
                     const uint32_t* ksigns, const float* knorms, const float* krnorms, const uint32_t* vcodes,
                     const float* vnorms, float scale, float* partials, float* out, void* stream, int partial_out,
                     int rn16);
int launch_decode_mma(const tq_ctx* hk, const tq_ctx* hv, const uint32_t* qfrag, const float* qscale, int B,
                      int Hq, int Hkv, int64_t T, int64_t kv_stride, const uint32_t* kcodes,
                      const uint32_t* ksigns, const float* knorms, const float* krnorms, const uint32_t* vcodes,
                      const float* vnorms, float scale, float* partials, float* out, void* stream,
                      int partial_out = 0, PagedCache pg = PagedCache());
// prefill (multi-query) attention on the tensor cores
bool prefill_supported(const tq_ctx* hk, const tq_ctx* hv, int Hq, int Hkv, int64_t kv_stride);
int prefill_splits(int B, int nq, int Hq, int Hkv, int64_t T, int sm_count);
size_t prefill_partials_bytes(int B, int nq, int Hq, int Hkv, int64_t T, int sm_count);
int launch_prefill(const tq_ctx* hk, const tq_ctx* hv, const float* qrot, const float* qproj, int B, int nq, int Hq,
                   int Hkv, int64_t T, int64_t kv_stride, const uint32_t* kcodes, const uint32_t* ksigns,
                   const float* knorms, const float* krnorms, const uint32_t* vcodes, const float* vnorms, float scale,
                   float* partials, float* out, void* stream);
// decode attention through whichever kernel fits; workspace layout owned here.
// partial_out: write the (acc[d] in the rotated value frame, m, l) record of
// every (batch, q-head) to out [B*Hq][d + 2] instead of the normalised output
size_t decode_workspace_bytes(const tq_ctx* hk, int B, int Hq, int Hkv, int64_t T);
int decode_dispatch(const tq_ctx* hk, const tq_ctx* hv, const void* q, int q_dtype, int B, int Hq, int Hkv,
                    int64_t T, int64_t kv_stride, const uint32_t* kcodes, const uint32_t* ksigns,
                    const float* knorms, const float* krnorms, const uint32_t* vcodes, const float* vnorms,
                    float scale, float* out, void* workspace, void* stream, int partial_out = 0,
                    PagedCache pg = PagedCache());
int launch_decode_simple(const tq_ctx* hk, const tq_ctx* hv, const float* qrot,
                         const float* qproj, int B, int Hq, int Hkv, int64_t T, int64_t kv_stride,
                         const uint32_t* kcodes, const uint32_t* ksigns, const float* knorms,
                         const float* krnorms, const uint32_t* vcodes, const float* vnorms,
                         float scale, int splits, float* partials, float* out, void* stream, int partial_out = 0,
                         PagedCache pg = PagedCache());

}  // namespace tqi
