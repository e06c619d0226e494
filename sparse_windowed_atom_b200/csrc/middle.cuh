// middle.cuh -- the middle of one forward pass, from the Q/K/V/value-gate projections
// to the fused tail (page "Local atom attention, encoder pooling and decoder
// skip/readout", Required behavior, bullets 4-18), with the Q/K/V/G/O intermediates of
// type WT (bf16 for bf16 workloads on the row-gather attention, float32 otherwise).
// Instantiated once per (storage type, WT) in middle_*.cu.
#pragma once

#include "host.cuh"

namespace atomenc {
namespace host {

template <typename Elt, typename WT>
void launch_middle(PassCtx<Elt> &c) {
  const Plan &pl = c.pl;
  const Dims &d = pl.d;
  const int64_t B = d.B, A = d.A, K = d.K, C = d.C, H = d.H, D = d.D, P = d.P, M = d.M,
                HD = H * D, R = B * A;
  const atomenc_inputs *in = c.in;
  const atomenc_outputs *out = c.out;
  const float eps = c.eps;
  const int64_t radius = c.radius;
  unsigned char *ws = c.ws;
  cudaStream_t st = c.st;
  Hooks &hk = c.hk;
  unsigned *status = c.status;
  uint8_t *usable = c.usable;
  const bool split = c.split, fuse_norm = c.fuse_norm;
  const unsigned row_blocks = c.row_blocks;
  Elt *xb = c.xb, *condb = c.condb, *gateb = c.gateb;
  auto F = [&](size_t off) { return c.F(off); };
  auto gemm_rows = [&](auto prod, size_t wpk, int64_t Mr, int64_t N, int64_t Kd, auto epi) {
    c.gemm_rows(prod, wpk, Mr, N, Kd, epi);
  };
  auto gemm = [&](auto *A_, int64_t lda, size_t wpk, int64_t Mr, int64_t N, int64_t Kd, auto epi) {
    c.gemm(A_, lda, wpk, Mr, N, Kd, epi);
  };
  auto norm_prod = [&](int64_t sc_off, int64_t sh_off, bool plus1) {
    return c.norm_prod(sc_off, sh_off, plus1);
  };
  WT *wq = reinterpret_cast<WT *>(ws + pl.o_q), *wk = reinterpret_cast<WT *>(ws + pl.o_k),
     *wv = reinterpret_cast<WT *>(ws + pl.o_v), *wg = reinterpret_cast<WT *>(ws + pl.o_g),
     *wo = reinterpret_cast<WT *>(ws + pl.o_o);
  // ---- projections (attention inputs fused into the operand when C <= 256)
  if (pl.af3) {
    EpiSplitT<WT> e0{{wq, wg, nullptr, nullptr}, {c.WF(pl.o_bq), nullptr, nullptr, nullptr}, HD};
    EpiSplitT<WT> e1{{wk, wv, nullptr, nullptr}, {nullptr, nullptr, nullptr, nullptr}, HD};
    if (fuse_norm) {
      gemm_rows(norm_prod(0, C, false), pl.k_qkv0, R, 2 * HD, C, e0);
      gemm_rows(norm_prod(2 * C, 3 * C, false), pl.k_qkv1, R, 2 * HD, C, e1);
    } else {
      gemm(F(pl.o_feat), 2 * C, pl.k_qkv0, R, 2 * HD, C, e0);
      gemm(F(pl.o_feat) + C, 2 * C, pl.k_qkv1, R, 2 * HD, C, e1);
    }
  } else {
    EpiSplitT<WT> e{{wq, wk, wv, wg}, {nullptr, nullptr, nullptr, nullptr}, HD};
    if (fuse_norm)
      gemm_rows(norm_prod(C, 0, true), pl.k_qkv0, R, 4 * HD, C, e);
    else
      gemm(F(pl.o_feat), C, pl.k_qkv0, R, 4 * HD, C, e);
    const uintptr_t rope_al = 4 * sizeof(Elt) - 1;
    const int rope_vec = ((reinterpret_cast<uintptr_t>(in->rope_cos.data) |
                           reinterpret_cast<uintptr_t>(in->rope_sin.data)) & rope_al) == 0;
    RopeArgs rp{R, H, D, eps, usable, in->rope_cos.data, in->rope_sin.data, wq, wk, rope_vec};
    if (D >= 8 && D <= 128 && (D & (D - 1)) == 0) {
      const int64_t warps = R;   // one per atom: its Q and K rows
      hk.launch(ATOMENC_KERNEL_ROWS, (k_qk_rope_warp<Elt, WT>), (unsigned)((warps + 7) / 8), 256, 0, st, rp);
    } else {
      const int64_t n = R * H * 2;
      hk.launch(ATOMENC_KERNEL_ROWS, (k_qk_rope<Elt>), (unsigned)((n + 255) / 256), 256, 0, st, rp);
    }
  }
  hk.mark(3, st);

  // ---- slot-gathered attention
  const int rad = radius < 0 ? -1 : (radius > INT_MAX ? INT_MAX : (int)radius);
  if (pl.rg) {
    RowAttnArgs ra2;
    ra2.B = (int)B; ra2.A = (int)A; ra2.K = (int)K; ra2.H = (int)H; ra2.D = (int)D; ra2.P = (int)P;
    ra2.radius = rad;
    ra2.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)D));
    ra2.eps = eps;
    ra2.QT = pl.rg_qt;
    ra2.tiles_per_b = (int)((A + pl.rg_qt - 1) / pl.rg_qt);
    ra2.ntiles = (int)B * ra2.tiles_per_b;
    ra2.stage_rows = pl.rg_stage_rows;
    ra2.qg_staged = pl.rg_qg ? 1 : 0;
    ra2.Q = wq; ra2.Kf = wk; ra2.Vf = wv; ra2.G = wg;
    ra2.key_index = static_cast<const int64_t *>(in->key_index.data);
    ra2.window = static_cast<const uint8_t *>(in->window_mask.data);
    ra2.usable = usable;
    ra2.pair = pl.af3 ? in->pair.data : nullptr;
    ra2.w_pair = c.WF(pl.o_wpair);
    ra2.attention = out->attention.data;
    ra2.O = wo;
    ra2.status = status;
    ra2.pair_vec = pl.af3 && P == 16 && (reinterpret_cast<uintptr_t>(in->pair.data) & 15) == 0;
    ra2.att_vec = (reinterpret_cast<uintptr_t>(out->attention.data) & 15) == 0;
    // persistent: one CTA per SM, each walking a contiguous range of tiles
    dim3 grid((unsigned)std::min<int64_t>(ra2.ntiles, pl.sms));
    auto go = [&](auto kern) {
      smem_limit(kern, pl.rg_smem);
      hk.launch(ATOMENC_KERNEL_ATTENTION, kern, grid, kRowAttnThreads, pl.rg_smem, st, ra2);
    };
    // the attention weights are written in the storage type: WT == Elt here
    if constexpr (std::is_same<WT, Elt>::value) {
#define ROWATTN(DH)                                                 \
if (D == DH) {                                                    \
  if (pl.af3) go(k_attn_rows<WT, 128, DH, true>);                 \
  else go(k_attn_rows<WT, 128, DH, false>);                       \
}
      ROWATTN(16) ROWATTN(32) ROWATTN(64)
#undef ROWATTN
    }
  } else {
    AttnArgs ag;
    ag.B = (int)B; ag.A = (int)A; ag.K = (int)K; ag.H = (int)H; ag.D = (int)D; ag.P = (int)P;
    ag.radius = rad;
    ag.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)D));
    ag.eps = eps;
    ag.QT = pl.QT; ag.DP = pl.DP; ag.kv_floats = pl.kv_floats;
    ag.kmagic = K > 1 ? (uint32_t)(((uint64_t)1 << 32) / (uint64_t)K + (((uint64_t)1 << 32) % (uint64_t)K != 0)) : 0u;
    ag.Q = F(pl.o_q); ag.Kf = F(pl.o_k); ag.Vf = F(pl.o_v); ag.G = F(pl.o_g);
    ag.key_index = static_cast<const int64_t *>(in->key_index.data);
    ag.window = static_cast<const uint8_t *>(in->window_mask.data);
    ag.usable = usable;
    ag.pair = pl.af3 ? in->pair.data : nullptr;
    ag.w_pair = c.WF(pl.o_wpair);
    ag.attention = out->attention.data;
    ag.O = F(pl.o_o);
    ag.status = status;
    dim3 grid((unsigned)((A + pl.QT - 1) / pl.QT), (unsigned)B);
    auto go = [&](auto kern) {
      smem_limit(kern, pl.attn_smem);
      hk.launch(ATOMENC_KERNEL_ATTENTION, kern, grid, attn_threads(pl.af3), pl.attn_smem, st, ag);
    };
    const int dm = D <= 8 ? 8 : D <= 16 ? 16 : D <= 32 ? 32 : 64;
    const bool multi = K > kChunk;
#define ATTN_D(DM)                                                          \
if (dm == DM) {                                                           \
  if (pl.af3)                                                             \
    multi ? go(k_slot_attention<Elt, DM, true, true>)                     \
          : go(k_slot_attention<Elt, DM, true, false>);                   \
  else                                                                    \
    multi ? go(k_slot_attention<Elt, DM, false, true>)                    \
          : go(k_slot_attention<Elt, DM, false, false>);                  \
}
    ATTN_D(8) ATTN_D(16) ATTN_D(32) ATTN_D(64)
#undef ATTN_D
  }

  hk.mark(4, st);

  // ---- out-projection + gated residual, transition norm, SwiGLU, gated residual + mask
  const Elt *gbuf = pl.af3 ? gateb : condb;
  const int64_t gld = pl.af3 ? 2 * C : 6 * C;
  const int64_t g0off = pl.af3 ? 0 : 2 * C, g1off = pl.af3 ? C : 5 * C;
  if (pl.fuse_tail) {
    TransArgs ta;
    ta.R = R; ta.HD = (int)HD; ta.M = (int)M;
    ta.O = wo; ta.x = xb;
    ta.g0 = gbuf + g0off; ta.g1 = gbuf + g1off; ta.g_ld = gld;
    ta.sc = condb + 4 * C; ta.sh = condb + (pl.af3 ? 5 : 3) * C; ta.cond_ld = 6 * C;
    ta.rms = pl.af3 ? 0 : 1; ta.plus1 = pl.af3 ? 0 : 1; ta.eps = eps;
    ta.usable = usable;
    ta.w_out = c.wb + pl.k_out; ta.w_ff1 = c.wb + pl.k_ff1; ta.w_ff2 = c.wb + pl.k_ff2;
    ta.hidden = out->hidden.data; ta.status = status;
    ta.xfer = F(pl.o_xfer); ta.xflag = reinterpret_cast<int *>(ws + pl.o_xflag);
    ta.peer_spin_limit = g_peer_spin_limit.load();
    ta.withhold_flag = g_peer_withhold.load();
    const size_t smem = trans_smem_bytes(split);
    const dim3 grid((unsigned)(((R + kUmmaBM - 1) / kUmmaBM) * (pl.tail_pair ? 2 : 1)));
    // the two CTAs of a row block exchange partials: launched as a 2-CTA cluster, so
    // that they are always resident at the same time
    auto go = [&](auto kern) {
      smem_limit(kern, smem);
      hk.launch_cluster(ATOMENC_KERNEL_TRANSITION, pl.tail_pair ? 2 : 1, kern, grid, kTransThreads,
                        smem, st, ta);
    };
    if constexpr (std::is_same<Elt, float>::value) {
      pl.tail_pair ? go(k_transition<true, Elt, true, WT>) : go(k_transition<true, Elt, false, WT>);
    } else {
      pl.tail_pair ? go(k_transition<false, Elt, true, WT>) : go(k_transition<false, Elt, false, WT>);
    }
  } else {
    gemm(static_cast<const WT *>(wo), HD, pl.k_out, R, C, HD,
         Quad<EpiResidual<Elt>>{{xb, gbuf, gld, g0off, C, F(pl.o_xp)}});
    TNormArgs tn{R, C, eps, pl.af3 ? 1 : 0, F(pl.o_xp), condb, F(pl.o_z)};
    hk.launch(ATOMENC_KERNEL_ROWS, (k_transition_norm<Elt>), row_blocks, 256, 0, st, tn);
    gemm(F(pl.o_z), C, pl.k_ff1, R, 2 * M, C, EpiSwiGLU{F(pl.o_h), M});
    gemm(F(pl.o_h), M, pl.k_ff2, R, C, M,
         Quad<EpiHidden<Elt>>{{F(pl.o_xp), gbuf, gld, g1off, C, usable,
                               static_cast<Elt *>(out->hidden.data)}});
  }
}

}  // namespace host
}  // namespace atomenc
