// Byte account of one decode step (host only).
//
// Paper form: the ByteCross README ("Overview"; "Usage: The byte account")
// counts the bytes a bandwidth-bound step re-reads -- the projection
// weights, fixed, and the KV cache, growing with the context n -- and
// derives the byte crossover (Equation 5) and the ideal speedup bound
// B_total / (B_total - dB).  The equations are not printed; these forms
// reproduce every printed value (n* = 44.6K / 74.3K / 104.0K for the
// Llama-3.1-8B shape at keep pairs 0.7/0.3, 0.5/0.3, 0.5/0.5; 1.60x at 128K
// with KV keep 0.3, which requires the LM head inside B_total).
//
// Implementation form: the bytes this library's step has to move, in closed
// form per mode: the rows of the kept channels of every projection, the LM
// head, the valid tokens of the kept pages, the key bounds of every page
// (kv modes), the append, norm gains, the embedding row and the logits.
// BC_SNAP reads the pages a once-after-prefill selection made at this
// context kept, plus a page the step's token opens, and no bounds; its paper
// form is the KV branch's.
#include "../../include/bytecross.h"

#include <math.h>
#include <algorithm>

static long long keep_rows(double ratio, long long n) {
  const double v = ceil(ratio * (double)n - 1e-9);
  return std::max(1LL, std::min(n, (long long)v));
}

extern "C" bc_status bc_byte_account(const bc_config* c, bc_mode mode, double rp, double rkv,
                                     long long n_ctx, int sinks, int recent, int page, bc_bytes* out) {
  if (!c || !out) return BC_EINVAL;
  if (c->n_layers < 1 || c->hidden < 1 || c->intermediate < 1 || c->n_heads < 1 || c->n_kv_heads < 1 ||
      c->head_dim < 1 || c->vocab < 1 || page < 1 || n_ctx < 0 || sinks < 0 || recent < 1)
    return BC_EINVAL;
  if (mode < BC_DENSE || mode > BC_MASKED) return BC_EINVAL;
  if (!(rp > 0 && rp <= 1) || !(rkv > 0 && rkv <= 1)) return BC_EINVAL;
  const bool act = mode == BC_ACT || mode == BC_BOTH;
  const bool kvs = mode == BC_KV || mode == BC_BOTH;
  const bool snap = mode == BC_SNAP;
  const double L = c->n_layers, d = c->hidden, f = c->intermediate;
  const double hq = (double)c->n_heads * c->head_dim, hkv = (double)c->n_kv_heads * c->head_dim;
  const double hd = c->head_dim, V = c->vocab;
  const double n = (double)n_ctx;

  // ---- paper form
  const double P_l = d * hq + 2 * d * hkv + hq * d + 3 * d * f;
  const double P_ff = 3 * d * f;
  out->weight_bytes = 2 * L * P_l;
  out->head_bytes = 2 * V * d;
  out->kv_bytes_per_token = 2 * L * 2 * hkv;
  out->dense_bytes = out->weight_bytes + out->head_bytes + n * out->kv_bytes_per_token;
  const double erp = act ? rp : 1.0, erkv = (kvs || snap) ? rkv : 1.0;
  out->saved_bytes = (1 - erp) * out->weight_bytes + (1 - erkv) * n * out->kv_bytes_per_token;
  out->bound = out->dense_bytes / (out->dense_bytes - out->saved_bytes);
  const double den = (1 - rkv) * 2 * hkv;
  out->n_star = den > 0 ? (1 - rp) * P_l / den : INFINITY;
  out->n_star_ff = den > 0 ? (1 - rp) * P_ff / den : INFINITY;

  // ---- implementation form
  const long long Hkv = c->n_kv_heads;
  const long long n_tok = n_ctx + 1;
  const long long P = (n_tok + page - 1) / page;
  auto kept = [&](long long pages) {
    const long long sink_end = std::min<long long>(sinks, pages);
    const long long rec_begin = std::max<long long>(pages - recent, 0);
    const long long forced = sink_end + (pages - std::max(rec_begin, sink_end));
    const long long want = std::min<long long>(pages, (long long)ceil(rkv * (double)pages - 1e-9));
    return std::max(forced, want);
  };
  long long K = P;
  if (kvs) K = kept(P);
  if (snap) {
    const long long P_sel = (std::max<long long>(n_ctx, 1) + page - 1) / page;
    K = kept(P_sel) + std::max<long long>(0, P - P_sel);
  }
  const long long qkv_cols = (long long)(hq + 2 * hkv);
  const long long kq = act ? keep_rows(rp, c->hidden) : c->hidden;
  const long long ko = act ? keep_rows(rp, (long long)hq) : (long long)hq;
  const long long kf = act ? keep_rows(rp, c->intermediate) : c->intermediate;
  const double row_bytes = 2.0 * ((double)kq * qkv_cols + (double)ko * d + (double)kq * 2 * f + (double)kf * d);
  out->impl_weight_bytes = L * row_bytes;
  out->impl_head_bytes = 2 * V * d;
  // the last page (partial, always kept: it is recent) holds n_tok - (P-1)*page tokens
  const long long last = n_tok - (P - 1) * page;
  const long long tokens_read = (kvs || snap) ? (K - 1) * page + last : n_tok;
  out->impl_kv_read_bytes = L * (double)Hkv * (double)tokens_read * 2 * hd * 2;
  out->impl_meta_read_bytes = kvs ? L * (double)Hkv * (double)P * 2 * hd * 2 : 0.0;
  out->impl_kv_write_bytes = L * (double)Hkv * (2 * hd * 2 + 2 * hd * 2);
  const long long slot = (n_tok - 1) % page;
  out->impl_other_bytes = L * (double)Hkv * (double)slot * hd * 2 + L * 2 * d * 2 + 2 * d + 2 * d + 4 * V;
  out->impl_total_bytes = out->impl_weight_bytes + out->impl_head_bytes + out->impl_kv_read_bytes +
                          out->impl_meta_read_bytes + out->impl_kv_write_bytes + out->impl_other_bytes;
  out->pages_total = P;
  out->pages_kept = K;
  return BC_OK;
}

// Batch crossover (ByteCross README, "Usage: The byte account"): a batch of
// `batch` sequences reads the union of its kept projection rows once
// (fraction union_keep of the weights) while every sequence saves its own
// KV bytes, so the two savings meet at
//   n = (1 - union_keep) P_l / (batch (1 - rkv) 2 Hkv hd) tokens.
extern "C" bc_status bc_crossover_batch(const bc_config* c, double union_keep, double rkv, int batch,
                                        double* n_star) {
  if (!c || !n_star) return BC_EINVAL;
  if (c->hidden < 1 || c->intermediate < 1 || c->n_heads < 1 || c->n_kv_heads < 1 || c->head_dim < 1)
    return BC_EINVAL;
  if (!(union_keep > 0 && union_keep <= 1) || !(rkv > 0 && rkv < 1) || batch < 1) return BC_EINVAL;
  const double d = c->hidden, f = c->intermediate;
  const double hq = (double)c->n_heads * c->head_dim, hkv = (double)c->n_kv_heads * c->head_dim;
  const double P_l = d * hq + 2 * d * hkv + hq * d + 3 * d * f;
  *n_star = (1 - union_keep) * P_l / ((double)batch * (1 - rkv) * 2 * hkv);
  return BC_OK;
}
