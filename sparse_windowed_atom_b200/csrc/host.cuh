// host.cuh -- host-side pieces shared by the translation units of the library: the
// pass plan, the launch hooks (programmatic serialization, clusters, per-kernel events),
// the pass context with the tensor-core GEMM launchers, and the declarations of the
// per-element-type launch sequences (defined in pass.cuh and middle.cuh, instantiated in
// pass_*.cu and middle_*.cu, so that the kernels of one pass compile in parallel).
#pragma once

#include <climits>
#include <cmath>
#include <cstring>
#include <algorithm>
#include <atomic>
#include <mutex>
#include <type_traits>
#include <utility>

#include "../../include/atomenc.h"
#include "attention.cuh"
#include "attn_rows.cuh"
#include "common.cuh"
#include "epilogues.cuh"
#include "gemm_umma.cuh"
#include "rows.cuh"
#include "transition.cuh"
#include "weights.cuh"

namespace atomenc {
namespace host {

constexpr int kMaxD = 64;
constexpr size_t kAttnSmemBudget = 210 * 1024;  // dynamic part: one CTA per SM, or per two (AF3) / 2 - 1 KB
constexpr size_t kRowAttnSmemBudget = 220 * 1024;  // dynamic part of the row-gather attention
constexpr int kMaxDevices = 64;

struct Dims {
  int64_t B = 0, A = 0, T = 0, K = 0, C = 0, S = 0, H = 0, D = 0, P = 0, M = 0, U = 0, V = 0;
};

constexpr size_t kImageHeader = 256;
// Modes of a pass: build the weight images in the workspace and run (the plain forward);
// build them into a prepared image only; run from a prepared image.
enum PassMode { kPassFull = 0, kPassPrepare = 1, kPassPrepared = 2 };

struct Plan {
  int style = 0, stage = 0, fdt = 0;
  bool af3 = false, enc = false, fuse_tail = false, tail_pair = false;
  Dims d;
  // workspace layout (byte offsets)
  size_t o_status, o_usable, o_xstats, o_cstats, o_first, o_last, o_tp, o_x, o_cond, o_gate, o_feat,
      o_q, o_k, o_v, o_g, o_o, o_xp, o_z, o_h, o_pool, o_xfer, o_xflag;
  size_t o_wread, o_bscale, o_brg, o_bq, o_wpair, o_rscale, o_rbias;
  // the weight region [o_wbase, bytes): panels and images built from the weights; a
  // prepared image holds it after a header of kImageHeader bytes
  size_t o_wbase = 0;
  // tensor-core images of the weight panels (bf16, hi[/lo])
  size_t k_cond, k_gate, k_qkv0, k_qkv1, k_out, k_ff1, k_ff2, k_pool, k_tok;
  size_t bytes = 0;
  // attention launch
  int QT = 0, DP = 0, kv_floats = 0;
  size_t attn_smem = 0;
  int sms = 148;                    // multiprocessors of the device the pass runs on
  // row-gather attention (k_attn_rows): H*D in {64, 128} ... see attn_rows.cuh; Q, K, V,
  // value-gate logits and the gated output are then kept in the storage type
  bool rg = false;
  int rg_qt = 0, rg_stage_rows = 0;
  bool rg_qg = false;               // row-gather attention stages the tile's Q and gate rows
  size_t rg_smem = 0;
  bool ws_bf16 = false;             // Q/K/V/G/O intermediates in bf16
};

// The key a prepared image carries: style, stage, storage type, the dimensions the images
// depend on (an FNV-1a hash of C, S, H, D, P, M, U, V) and the weight region's size.
inline void image_key(const Plan &pl, int (&key)[kImageKeyWords]) {
  const Dims &d = pl.d;
  key[0] = 0x61656e63;
  key[1] = pl.style | (pl.stage << 4) | (pl.fdt << 8);
  uint32_t h = 2166136261u;
  const int64_t dims[8] = {d.C, d.S, d.H, d.D, d.P, d.M, d.U, d.V};
  for (int64_t v : dims) {
    h = (h ^ (uint32_t)v) * 16777619u;
    h = (h ^ (uint32_t)(v >> 32)) * 16777619u;
  }
  key[2] = (int)h;
  key[3] = (int)(pl.bytes - pl.o_wbase);
}

// Raise a kernel's dynamic shared-memory limit once per (kernel, device), and again only
// if a larger size is asked for: the attribute outlives the call, so repeating it on
// every forward would only add host time (defined in atomenc.cu).
cudaError_t smem_limit_fn(const void *fn, size_t bytes);
template <typename... KP>
inline cudaError_t smem_limit(void (*kern)(KP...), size_t bytes) {
  return smem_limit_fn(reinterpret_cast<const void *>(kern), bytes);
}

struct Hooks {
  cudaEvent_t const *ev = nullptr;  // ATOMENC_NUM_PHASES + 1 events, or null
  cudaEvent_t const *kev = nullptr; // traced: one event before the pass and one per launch
  int n_kev = 0;
  int *kinds = nullptr;             // traced: enum atomenc_kernel_kind per launch
  int launches = 0;
  cudaError_t err = cudaSuccess;    // first launch failure
  bool overflow = false;            // traced: more launches than events
  void mark(int i, cudaStream_t st) const {
    if (ev) cudaEventRecord(ev[i], st);
  }
  void begin(cudaStream_t st) {
    if (kev && n_kev > 0) cudaEventRecord(kev[0], st);
  }
  // Every kernel is launched here, with programmatic stream serialization: it may be
  // scheduled while its predecessor finishes and waits for it in pdl_enter(). A
  // cluster size of 2 launches the grid as CTA pairs that the hardware schedules
  // together.
  template <typename... KP, typename... Args>
  void launch(int kind, void (*kern)(KP...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
              Args &&...args) {
    launch_cluster(kind, 1, kern, grid, block, smem, st, std::forward<Args>(args)...);
  }
  template <typename... KP, typename... Args>
  void launch_cluster(int kind, int cluster, void (*kern)(KP...), dim3 grid, dim3 block,
                      size_t smem, cudaStream_t st, Args &&...args) {
    cudaLaunchAttribute at[2];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    int nat = 1;
    if (cluster > 1) {
      at[1].id = cudaLaunchAttributeClusterDimension;
      at[1].val.clusterDim.x = (unsigned)cluster;
      at[1].val.clusterDim.y = 1;
      at[1].val.clusterDim.z = 1;
      nat = 2;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = at;
    cfg.numAttrs = nat;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
    if (e != cudaSuccess && err == cudaSuccess) err = e;
    if (kev) {
      if (launches + 1 < n_kev) {
        cudaEventRecord(kev[launches + 1], st);
        if (kinds) kinds[launches] = kind;
      } else {
        overflow = true;
      }
    }
    ++launches;
  }
};

// Test hook for the bounded wait of the paired transition CTAs (see
// atomenc_debug_peer_wait): poll limit, and whether the partials' flags are withheld.
extern std::atomic<uint32_t> g_peer_spin_limit;
extern std::atomic<int> g_peer_withhold;

// Everything one pass's launches share.
template <typename Elt>
struct PassCtx {
  const Plan &pl;
  const atomenc_inputs *in;
  const atomenc_params *p;
  const atomenc_outputs *out;
  float eps;
  int64_t radius;
  unsigned char *ws;
  cudaStream_t st;
  Hooks &hk;
  unsigned *status;
  uint8_t *usable;
  bool split;           // float32 workload: three bf16 products per product
  bool fuse_norm;       // the row norm of x is formed inside the projection operand
  unsigned row_blocks;  // 256-thread blocks of the warp-per-row kernels
  Elt *xb, *condb, *gateb, *poolb;   // intermediates in the storage type
  unsigned char *wb;    // base of the weight-region offsets (the workspace, or a prepared image)
  float *F(size_t off) const { return reinterpret_cast<float *>(ws + off); }
  float *WF(size_t off) const { return reinterpret_cast<float *>(wb + off); }

  // out = epi(A' @ W) on the tensor cores, W given by its packed image and A' produced by
  // `prod` (A itself, or a row normalisation fused into the operand); K <= 256
  template <class P, class E>
  void gemm_rows(P prod, size_t wpk, int64_t Mr, int64_t N, int64_t Kd, E epi) {
    const int64_t mt = (Mr + kUmmaBM - 1) / kUmmaBM, nt = (N + kUmmaBN - 1) / kUmmaBN;
    // enough row blocks for every SM (a formed operand: three per SM, so that forming the
    // next block's operand overlaps enough tiles): the persistent kernel (one CTA per SM,
    // the next block's operand formed while the current one's tiles run)
    if (!split && mt >= (P::kLight ? 1 : 3) * (int64_t)pl.sms) {
      constexpr int EW = P::kEpiWarps;
      const int nslot = rows_p_slots(Kd, EW);
      const size_t smem = rows_p_smem_bytes(Kd, nslot, EW);
      if (smem <= kRowsSmemBudget) {
        smem_limit(k_gemm_rows_p<P, E, EW>, smem);
        hk.launch(ATOMENC_KERNEL_GEMM, (k_gemm_rows_p<P, E, EW>), dim3((unsigned)pl.sms), kRowsPThreads,
                  smem, st, prod, wb + wpk, Mr, N, Kd, nslot, epi, status);
        return;
      }
    }
    const int64_t want = (pl.sms + mt - 1) / mt;          // CTAs per row block to fill the GPU
    const int64_t sp = want < nt ? want : nt;
    const int per = (int)((nt + sp - 1) / sp);
    dim3 grid((unsigned)((nt + per - 1) / per), (unsigned)mt);
    const int nkc = (int)((Kd + kUmmaBK - 1) / kUmmaBK);
    const int nslot = rows_slots(Kd, split, per * nkc);
    const size_t smem = rows_smem_bytes(Kd, split, nslot);
    if (split) {
      smem_limit(k_gemm_rows<P, true, E>, smem);
      hk.launch(ATOMENC_KERNEL_GEMM, (k_gemm_rows<P, true, E>), grid, kRowsThreads, smem, st, prod, wb + wpk, Mr, N, Kd, per, nslot, epi, status);
    } else {
      smem_limit(k_gemm_rows<P, false, E>, smem);
      hk.launch(ATOMENC_KERNEL_GEMM, (k_gemm_rows<P, false, E>), grid, kRowsThreads, smem, st, prod, wb + wpk, Mr, N, Kd, per, nslot, epi, status);
    }
  }
  // out = epi(A @ W): the row-block kernel for K <= 256, else the streaming kernel
  template <typename TA, class E>
  void gemm(const TA *A_, int64_t lda, size_t wpk, int64_t Mr, int64_t N, int64_t Kd, E epi) {
    if (Kd <= kRowsKMax) {
      gemm_rows(ProdPlain<TA>{A_, lda, Mr, Kd}, wpk, Mr, N, Kd, epi);
      return;
    }
    dim3 grid((unsigned)((N + kUmmaBN - 1) / kUmmaBN), (unsigned)((Mr + kUmmaBM - 1) / kUmmaBM));
    const size_t smem = umma_smem_bytes(split);
    if (split) {
      smem_limit(k_gemm_umma<TA, true, E>, smem);
      hk.launch(ATOMENC_KERNEL_GEMM, (k_gemm_umma<TA, true, E>), grid, kUmmaThreads, smem, st, A_, lda, wb + wpk, Mr, N, Kd, epi, status);
    } else {
      smem_limit(k_gemm_umma<TA, false, E>, smem);
      hk.launch(ATOMENC_KERNEL_GEMM, (k_gemm_umma<TA, false, E>), grid, kUmmaThreads, smem, st, A_, lda, wb + wpk, Mr, N, Kd, epi, status);
    }
  }
  // the conditioning-modulated row norm of x fused into a projection's operand
  ProdNormT<Elt> norm_prod(int64_t sc_off, int64_t sh_off, bool plus1) const {
    return ProdNormT<Elt>{xb, F(pl.o_xstats), condb, pl.d.B * pl.d.A, pl.d.C, 6 * pl.d.C, sc_off,
                          sh_off, plus1 ? 1 : 0};
  }
};

// The launch sequence of one pass (pass.cuh), and its middle from the projections to the
// fused tail with the Q/K/V/G/O intermediates of type WT (middle.cuh).
template <typename Elt>
int launch_all(const Plan &pl, const atomenc_inputs *in, const atomenc_params *p, float eps,
               int64_t radius, const atomenc_outputs *out, unsigned char *ws, cudaStream_t st,
               Hooks &hk, int mode = kPassFull, unsigned char *image = nullptr);
template <typename Elt, typename WT>
void launch_middle(PassCtx<Elt> &c);

}  // namespace host
}  // namespace atomenc
