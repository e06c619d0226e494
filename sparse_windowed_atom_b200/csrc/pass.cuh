// pass.cuh -- the launch sequence of one forward pass (page "Local atom attention,
// encoder pooling and decoder skip/readout", Required behavior, in its order):
// weight images, usability + sanitisation + residual start (bullets 2-3), conditioning
// (AF3 bullets 7, 9; ESMFold2 bullet 10), then the middle (middle.cuh: projections,
// attention, out-projection and transition, bullets 4-18), then encoder pooling or
// decoder readout (bullets 18-20). Instantiated once per storage type (pass_*.cu).
#pragma once

#include "host.cuh"

namespace atomenc {
namespace host {

template <typename Elt>
int launch_all(const Plan &pl, const atomenc_inputs *in, const atomenc_params *p,
               float eps, int64_t radius, const atomenc_outputs *out, unsigned char *ws,
               cudaStream_t st, Hooks &hk, int mode, unsigned char *image) {
  const Dims &d = pl.d;
  const int64_t B = d.B, A = d.A, T = d.T, C = d.C, S = d.S, H = d.H, D = d.D,
                P = d.P, M = d.M, U = d.U, V = d.V, HD = H * D, R = B * A;
  auto F = [&](size_t off) { return reinterpret_cast<float *>(ws + off); };
  // weight-region offsets resolve against the workspace, or against a prepared image
  // (whose region starts after its header)
  unsigned char *wb = mode == kPassFull ? ws
                                        : reinterpret_cast<unsigned char *>(
                                              reinterpret_cast<uintptr_t>(image) + kImageHeader - pl.o_wbase);
  auto WF = [&](size_t off) { return reinterpret_cast<float *>(wb + off); };
  unsigned *status = mode == kPassPrepare ? nullptr : reinterpret_cast<unsigned *>(ws + pl.o_status);
  uint8_t *usable = ws + pl.o_usable;
  int *first = reinterpret_cast<int *>(ws + pl.o_first);
  int *last = reinterpret_cast<int *>(ws + pl.o_last);

  hk.mark(0, st);

  // ---- one launch: tensor-core images of the projection weights (built from the
  // caller's tensors), small float32 panels, status and token-range resets
  WeightJobs wj;
  std::memset(&wj, 0, sizeof(wj));
  const size_t es = sizeof(Elt);
  auto elt = [&](const atomenc_tensor &t, size_t off) -> const void * {
    return t.data ? static_cast<const unsigned char *>(t.data) + off * es : nullptr;
  };
  auto copy = [&](const atomenc_tensor &src, size_t src_off, int64_t rows, int64_t cols, size_t dst_off,
                  int64_t dst_ld, int64_t col0, const atomenc_tensor *rowscale, size_t rs_off) {
    CopyJob &j = wj.copy[wj.ncopy++];
    j.src = elt(src, src_off);
    j.rowscale = rowscale ? elt(*rowscale, rs_off) : nullptr;
    j.dst = WF(dst_off);
    j.rows = (int32_t)rows;
    j.cols = (int32_t)cols;
    j.dst_ld = (int32_t)dst_ld;
    j.dst_col0 = (int32_t)col0;
    j.dst_cstride = 1;
  };
  const bool split = pl.fdt == ATOMENC_F32;
  auto pack = [&](size_t dst, int64_t Kd, int64_t N) -> PackJob & {
    PackJob &j = wj.pack[wj.npack++];
    j.dst = wb + dst;
    j.K = (int32_t)Kd;
    j.N = (int32_t)N;
    j.split = split ? 1 : 0;
    return j;
  };
  auto seg = [&](PackJob &j, const atomenc_tensor &src, size_t src_off, int64_t cols, int64_t col0,
                 int cshift, const atomenc_tensor *rowscale, size_t rs_off) {
    PackSeg &g = j.seg[j.nseg++];
    g.src = elt(src, src_off);
    g.rowscale = rowscale ? elt(*rowscale, rs_off) : nullptr;
    g.cols = (int32_t)cols;
    g.col0 = (int32_t)col0;
    g.cshift = cshift;
  };
  if (mode != kPassPrepared) {   // the images and panels (a prepared image has them)
  if (pl.af3) {
    PackJob &jc = pack(pl.k_cond, S, 6 * C);
    for (int jj = 0; jj < 3; ++jj) {
      seg(jc, p->w_scale, (size_t)jj * S * C, C, 2 * jj * C, 0, &p->cond_scale, (size_t)jj * S);
      seg(jc, p->w_shift, (size_t)jj * S * C, C, 2 * jj * C + C, 0, &p->cond_scale, (size_t)jj * S);
    }
    PackJob &jg = pack(pl.k_gate, S, 2 * C);
    seg(jg, p->w_residual_gate, 0, C, 0, 0, nullptr, 0);
    seg(jg, p->w_residual_gate, (size_t)S * C, C, C, 0, nullptr, 0);
    PackJob &j0 = pack(pl.k_qkv0, C, 2 * HD);
    seg(j0, p->w_q, 0, HD, 0, 0, nullptr, 0);
    seg(j0, p->w_value_gate, 0, HD, HD, 0, nullptr, 0);
    PackJob &j1 = pack(pl.k_qkv1, C, 2 * HD);
    seg(j1, p->w_k, 0, HD, 0, 0, nullptr, 0);
    seg(j1, p->w_v, 0, HD, HD, 0, nullptr, 0);
    copy(p->b_scale, 0, 1, 3 * C, pl.o_bscale, 3 * C, 0, nullptr, 0);
    copy(p->b_residual_gate, 0, 1, 2 * C, pl.o_brg, 2 * C, 0, nullptr, 0);
    copy(p->b_q, 0, 1, HD, pl.o_bq, HD, 0, nullptr, 0);
    copy(p->w_pair, 0, P, H, pl.o_wpair, H, 0, &p->pair_scale, 0);
  } else {
    seg(pack(pl.k_cond, S, 6 * C), p->w_mod, 0, 6 * C, 0, 0, nullptr, 0);
    PackJob &j0 = pack(pl.k_qkv0, C, 4 * HD);
    seg(j0, p->w_q, 0, HD, 0, 0, nullptr, 0);
    seg(j0, p->w_k, 0, HD, HD, 0, nullptr, 0);
    seg(j0, p->w_v, 0, HD, 2 * HD, 0, nullptr, 0);
    seg(j0, p->w_value_gate, 0, HD, 3 * HD, 0, nullptr, 0);
  }
  seg(pack(pl.k_out, HD, C), p->w_attention_out, 0, C, 0, 0, nullptr, 0);
  PackJob &jf = pack(pl.k_ff1, C, 2 * M);
  seg(jf, p->w_ff_gate, 0, M, 0, 1, nullptr, 0);
  seg(jf, p->w_ff_up, 0, M, 1, 1, nullptr, 0);
  seg(pack(pl.k_ff2, M, C), p->w_ff_out, 0, C, 0, 0, nullptr, 0);
  if (pl.enc) {
    seg(pack(pl.k_pool, C, U), p->w_pool, 0, U, 0, 0, nullptr, 0);
  } else {
    seg(pack(pl.k_tok, V, C), p->w_token, 0, C, 0, 0, nullptr, 0);
    copy(p->readout_scale, 0, 1, C, pl.o_rscale, C, 0, nullptr, 0);
    if (!pl.af3) copy(p->readout_bias, 0, 1, C, pl.o_rbias, C, 0, nullptr, 0);
    copy(p->w_readout, 0, C, 3, pl.o_wread, 3, 0, nullptr, 0);
  }
  }
  // the image key: style, stage, storage type and every dimension the images depend on
  image_key(pl, wj.key);
  if (mode == kPassPrepare) {
    wj.key_out = reinterpret_cast<int *>(image);
    hk.launch(ATOMENC_KERNEL_PREP, (k_prep_weights<Elt>), dim3(kPrepBlocksPerJob, wj.ncopy + wj.npack), 256, 0, st, wj);
    if (hk.err != cudaSuccess) return ATOMENC_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? ATOMENC_OK : ATOMENC_ERR_CUDA;
  }
  if (mode == kPassPrepared) wj.key_in = reinterpret_cast<const int *>(image);
  wj.status = status;   // reset (bit 8 when a prepared image does not match)
  if (pl.tail_pair)
    wj.fill[wj.nfill++] = FillJob{reinterpret_cast<int *>(ws + pl.o_xflag), 2 * ((R + kUmmaBM - 1) / kUmmaBM), 0, 0};
  if (pl.enc) {
    wj.fill[wj.nfill++] = FillJob{first, B * T, INT_MAX, 0};
    wj.fill[wj.nfill++] = FillJob{last, B * T, -1, 0};
  }
  hk.launch(ATOMENC_KERNEL_PREP, (k_prep_weights<Elt>), dim3(kPrepBlocksPerJob, std::max(wj.ncopy + wj.npack + wj.nfill, 1)), 256, 0, st, wj);

  const bool fuse_norm = C <= kRowsKMax;
  const int rows_per_block = 8;  // warps per 256-thread block for warp-per-row kernels
  const unsigned row_blocks = (unsigned)((R + rows_per_block - 1) / rows_per_block);
  Elt *xb = reinterpret_cast<Elt *>(ws + pl.o_x), *condb = reinterpret_cast<Elt *>(ws + pl.o_cond),
      *gateb = reinterpret_cast<Elt *>(ws + pl.o_gate), *poolb = reinterpret_cast<Elt *>(ws + pl.o_pool);
  PassCtx<Elt> c{pl, in, p, out, eps, radius, ws, st, hk, status, usable, split, fuse_norm,
                 row_blocks, xb, condb, gateb, poolb, wb};

  // ---- decoder: token @ w_token, gathered per atom in the row pass
  if (!pl.enc)
    c.gemm(static_cast<const Elt *>(in->token.data), V, pl.k_tok, B * T, C, V,
         QuadStore<float>{F(pl.o_tp), C});

  // ---- usable, sanitised residual start, normalised condition
  RowsArgs ra;
  ra.B = B; ra.A = A; ra.T = T; ra.C = C; ra.S = S; ra.eps = eps;
  ra.af3 = pl.af3; ra.decoder = !pl.enc; ra.encoder = pl.enc;
  ra.atom = in->atom.data; ra.condition = in->condition.data;
  ra.valid = static_cast<const uint8_t *>(in->valid.data);
  ra.token_valid = static_cast<const uint8_t *>(in->token_valid.data);
  ra.att = static_cast<const int64_t *>(in->atom_to_token.data);
  ra.token_proj = F(pl.o_tp);
  ra.usable = usable; ra.x = xb; ra.xstats = F(pl.o_xstats); ra.cstats = F(pl.o_cstats);
  ra.tok_first = first; ra.tok_last = last;
  {
    const uintptr_t al = sizeof(Elt) == 4 ? 15 : 7;   // 4-element loads of atom / condition rows
    const bool reg = C % 4 == 0 && S % 4 == 0 && C <= 256 && S <= 256 &&
                     ((reinterpret_cast<uintptr_t>(in->atom.data) | reinterpret_cast<uintptr_t>(in->condition.data)) & al) == 0;
    if (reg)
      hk.launch(ATOMENC_KERNEL_ROWS, (k_rows_prep_reg<Elt>), dim3((unsigned)((A + 7) / 8), (unsigned)B), 256, 0,
                st, ra);
    else
      hk.launch(ATOMENC_KERNEL_ROWS, (k_rows_prep<Elt>), row_blocks, 256, 0, st, ra);
  }
  hk.mark(1, st);

  // ---- conditioning: the operand (LN(c), raw c or SiLU(c) of the sanitised condition)
  // is formed from the caller's condition rows inside the product
  const Elt *cin = static_cast<const Elt *>(in->condition.data);
  if (pl.af3) {
    c.gemm_rows(ProdCond<Elt, 2>{cin, usable, F(pl.o_cstats), R, S}, pl.k_cond, R, 6 * C, S,
              EpiCondAF3<Elt>{condb, WF(pl.o_bscale), C});
    c.gemm_rows(ProdCond<Elt, 0>{cin, usable, nullptr, R, S}, pl.k_gate, R, 2 * C, S,
              EpiGateAF3<Elt>{gateb, WF(pl.o_brg), C});
  } else {
    c.gemm_rows(ProdCond<Elt, 1>{cin, usable, nullptr, R, S}, pl.k_cond, R, 6 * C, S,
              QuadStore<Elt>{condb, 6 * C});
  }
  hk.mark(2, st);
  if (!fuse_norm) {
    FeatArgs fa{R, C, eps, pl.af3 ? 1 : 0, xb, condb, F(pl.o_feat)};
    hk.launch(ATOMENC_KERNEL_ROWS, (k_features<Elt>), row_blocks, 256, 0, st, fa);
  }

  // ---- projections .. fused tail (middle.cuh)
  if constexpr (std::is_same<Elt, __nv_bfloat16>::value) {
    if (pl.ws_bf16)
      launch_middle<Elt, __nv_bfloat16>(c);
    else
      launch_middle<Elt, float>(c);
  } else {
    launch_middle<Elt, float>(c);
  }

  hk.mark(5, st);

  // ---- boundary, read from the hidden output itself
  const Elt *hid = static_cast<const Elt *>(out->hidden.data);
  if (pl.enc) {
    c.gemm(hid, C, pl.k_pool, R, U, C, QuadRelu<Elt>{poolb, U});
    PoolArgs pa{B, A, T, U, usable, static_cast<const int64_t *>(in->atom_to_token.data), first,
                last, poolb, out->token_output.data};
    const int vec_out = (reinterpret_cast<uintptr_t>(out->token_output.data) & (4 * sizeof(Elt) - 1)) == 0;
    const dim3 tok_blocks((unsigned)((T + 7) / 8), (unsigned)B);   // k_token_mean_warp
    if (U % 4 == 0 && U <= 128)
      hk.launch(ATOMENC_KERNEL_POOL, (k_token_mean_warp<Elt, 1>), tok_blocks, 256, 0, st, pa, vec_out);
    else if (U % 4 == 0 && U <= 256)
      hk.launch(ATOMENC_KERNEL_POOL, (k_token_mean_warp<Elt, 2>), tok_blocks, 256, 0, st, pa, vec_out);
    else if (U % 4 == 0 && U <= 384)
      hk.launch(ATOMENC_KERNEL_POOL, (k_token_mean_warp<Elt, 3>), tok_blocks, 256, 0, st, pa, vec_out);
    else if (U % 4 == 0 && U <= 512)
      hk.launch(ATOMENC_KERNEL_POOL, (k_token_mean_warp<Elt, 4>), tok_blocks, 256, 0, st, pa, vec_out);
    else
      hk.launch(ATOMENC_KERNEL_POOL, (k_token_mean<Elt>), (unsigned)(B * T), kPoolThreads, 0, st, pa);
  } else {
    ReadoutArgs rd{R, C, eps, pl.af3 ? 0 : 1, usable, hid, WF(pl.o_rscale), WF(pl.o_rbias),
                   WF(pl.o_wread), out->position_update.data};
    hk.launch(ATOMENC_KERNEL_ROWS, (k_readout<Elt>), row_blocks, 256, 0, st, rd);
  }
  hk.mark(6, st);
  if (hk.err != cudaSuccess) return ATOMENC_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? ATOMENC_OK : ATOMENC_ERR_CUDA;
}


}  // namespace host
}  // namespace atomenc
