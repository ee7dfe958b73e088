// Oracle for the MoE layer forward (Gate -> Scatter -> Expert Compute -> Gather).
//
// TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the benchmark's CPU
// baseline may load this library.  It shares no code, header, table or constant with the
// CUDA library: every step is written out here, plainly and slowly, single-threaded.
//
// Arithmetic: inputs are widened exactly to double (float32 as is, bfloat16 by placing its
// bits in the top half of a float32, int8 weights dequantised as the float32 product
// s[o] * q[o][i], int4 weights as the float32 product s[o][i / 128] * q[o][i]); every dot
// product and sum is accumulated in double in ascending index order and rounded to float32
// once.  Results are float32.
//
// The pages describing the method (the "Colibri" MoE engine) are cited by address and
// section:
//   [0539edu]  www.0539edu.com/news/4774449   (engine overview)
//   [mhpq]     www.mhpq.cn/news/563172        (routing kernel, fixed-stride experts)
//   [hotelren] www.hotelren.com/news/4731937  (six-step MoE flow, router, combine)
//   [trdm]     www.trdm.cn/news/555962        (grouping tokens by expert)
//   [pptc]     www.pptc.cn/news/100465        (expert_offsets, [batch][k] routing layout)
//
// Readings taken where the pages are silent or disagree:
//   * weights are the softmax over all E logits renormalised over the k chosen, which is
//     exp(l_j - l_0) / sum_j' exp(l_j' - l_0) over the chosen set; the raw-logit variant
//     ([hotelren] §3.2: no softmax) takes the chosen logits themselves as the weights;
//   * the clamp variant limits the logits to [-50, 50] before selection and weighting, so
//     logits beyond 50 tie and the tie rule below decides;
//   * ties in the logits go to the lower expert index;
//   * slot 0 holds the largest logit;
//   * the expert FFN is SwiGLU: W2 (silu(W1 x) * (W3 x)), no biases;
//   * within one expert, rows are in ascending token order;
//   * the optional shared expert is a SwiGLU FFN added with weight 1;
//   * int4 weights ([mhpq] §4.2: INT4 packed in INT32, group-wise quantisation with group size
//     128; [trdm] §6.1: two 4-bit weights per byte, unpacked at compute time): element 2j of a
//     row sits in the low nibble of byte j and element 2j + 1 in the high nibble (so the eight
//     elements of a little-endian int32 run from its lowest nibble up), each a two's-complement
//     value in [-8, 7]; symmetric, no zero point (the int8 quantiser of [0539edu] §3.1 has
//     none); one fp32 scale per output row and group of 128 consecutive inputs, stored
//     group-major ([cols / 128][rows] per matrix: the scales of one group's rows are adjacent;
//     the pages do not fix this layout).
//
// Parity pins: see tests/test_oracle_pins.py (brute force, closed forms, invariants).

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

namespace {

enum { ORC_F32 = 0, ORC_BF16 = 1, ORC_I8 = 2, ORC_I4 = 3 };
constexpr int kI4Group = 128;  // inputs per int4 scale group
enum { ORC_OK = 0, ORC_EARG = -1, ORC_ENONFINITE = -2 };
// Router variants: clamp the logits to [-50, 50] ([0539edu] §5.2, the gate-softmax clip
// option against overflow); use the chosen raw logits as the combine weights, no softmax
// ([hotelren] §3.2).
enum { ORC_ROUTER_CLAMP = 1, ORC_ROUTER_RAW = 2 };

// Exact widening of one stored element to double.
inline double widen(const void* p, int dtype, int64_t i) {
  if (dtype == ORC_F32) return (double)((const float*)p)[i];
  if (dtype == ORC_BF16) {
    uint32_t bits = (uint32_t)((const uint16_t*)p)[i] << 16;
    float v;
    std::memcpy(&v, &bits, 4);
    return (double)v;
  }
  return (double)((const int8_t*)p)[i];
}

// The signed 4-bit value stored at element index n of a packed int4 buffer.
inline int int4_at(const void* w, int64_t n) {
  const uint8_t byte = ((const uint8_t*)w)[n >> 1];
  const int nib = (n & 1) ? (byte >> 4) : (byte & 0xF);
  return nib >= 8 ? nib - 16 : nib;
}

// One weight matrix element W[o][i] of a [rows, cols] row-major matrix at element offset
// `base` of the expert buffer.  For int8 storage the element is s[o] * q[o][i] rounded to
// float32 ("per-output-channel fp32 scale, dequantised in the kernel"); for int4 storage it is
// s[i / 128][o] * q[o][i] with the matrix's scales [cols / 128][rows].
inline double weight(const void* w, int wdt, int64_t base, int64_t rows, int64_t cols, int64_t o, int64_t i,
                     const float* scale) {
  if (wdt == ORC_I8) {
    float deq = scale[o] * (float)((const int8_t*)w)[base + o * cols + i];
    return (double)deq;
  }
  if (wdt == ORC_I4) {
    float deq = scale[(i / kI4Group) * rows + o] * (float)int4_at(w, base + o * cols + i);
    return (double)deq;
  }
  return widen(w, wdt, base + o * cols + i);
}

// Scales of one expert: int8 [f | f | d] per output channel, int4 [d/128][f] | [d/128][f] |
// [f/128][d] per input group and output channel.
inline int64_t expert_scale_count(int wdt, int d, int f) {
  if (wdt == ORC_I8) return 2 * (int64_t)f + d;
  if (wdt == ORC_I4) return 3 * (int64_t)d * f / kI4Group;
  return 0;
}
inline bool quantised(int wdt) { return wdt == ORC_I8 || wdt == ORC_I4; }

// SwiGLU feed-forward of one input row through one expert whose three matrices start at
// element `base` of buffer `w`: W1[f][d] (gate), W3[f][d] (up), W2[d][f] (down).
// [hotelren] §2.1 (six steps: each chosen expert is an FFN applied to the token), SwiGLU form
// as the workloads state.  `scales` (int8 / int4 only) holds the expert's scales in the layout
// of expert_scale_count.
bool expert_ffn(const double* xrow, int d, int f, const void* w, int wdt, int64_t base,
                const float* scales, float* yrow) {
  std::vector<float> h(f);
  const int64_t w1 = base, w3 = base + (int64_t)f * d, w2 = base + 2 * (int64_t)f * d;
  const int64_t s3_off = wdt == ORC_I4 ? (int64_t)f * d / kI4Group : f;
  const float* s1 = scales ? scales : nullptr;
  const float* s3 = scales ? scales + s3_off : nullptr;
  const float* s2 = scales ? scales + 2 * s3_off : nullptr;
  for (int o = 0; o < f; ++o) {
    double g = 0.0, u = 0.0;
    for (int i = 0; i < d; ++i) {
      g += weight(w, wdt, w1, f, d, o, i, s1) * xrow[i];
      u += weight(w, wdt, w3, f, d, o, i, s3) * xrow[i];
    }
    const double gf = (double)(float)g, uf = (double)(float)u;
    const double hv = gf / (1.0 + std::exp(-gf)) * uf;  // silu(g) * u
    h[o] = (float)hv;
    if (!std::isfinite(h[o])) return false;
  }
  for (int o = 0; o < d; ++o) {
    double acc = 0.0;
    for (int i = 0; i < f; ++i) acc += weight(w, wdt, w2, d, f, o, i, s2) * (double)h[i];
    yrow[o] = (float)acc;
    if (!std::isfinite(yrow[o])) return false;
  }
  return true;
}

}  // namespace

extern "C" {

// Step 1, router logits: l[t][e] = b[e] + sum_i x[t][i] * Wr[e][i].
// [0539edu] §2.1 (gate output of shape [batch, seq_len, num_experts], then softmax and
// top-k); [hotelren] §3.2 (linear projection input @ router_weight + router_bias).
// With ORC_ROUTER_CLAMP in `flags` each logit is then limited to [-50, 50] ([0539edu] §5.2).
int oracle_router_logits(const void* x, int act, int T, int d, const void* wr, const float* b,
                         int E, int flags, float* logits) {
  if (T < 0 || d <= 0 || E <= 0 || (T > 0 && (!x || !wr || !logits))) return ORC_EARG;
  if (flags & ~(ORC_ROUTER_CLAMP | ORC_ROUTER_RAW)) return ORC_EARG;
  for (int t = 0; t < T; ++t) {
    for (int e = 0; e < E; ++e) {
      double acc = 0.0;
      for (int i = 0; i < d; ++i)
        acc += widen(x, act, (int64_t)t * d + i) * widen(wr, act, (int64_t)e * d + i);
      if (b) acc += (double)b[e];
      if (flags & ORC_ROUTER_CLAMP) acc = std::min(50.0, std::max(-50.0, acc));
      logits[(int64_t)t * E + e] = (float)acc;
      if (!std::isfinite(logits[(int64_t)t * E + e])) return ORC_ENONFINITE;
    }
  }
  return ORC_OK;
}

// Step 2/3 weights for a given selection: w_j = exp(l_j - l_0) / sum_j' exp(l_j' - l_0),
// which equals the softmax over all E renormalised over the chosen k (the common
// normaliser cancels).  [0539edu] §2.1 softmax then top-k; renormalised over the chosen k.
// With ORC_ROUTER_RAW in `flags`, w_j = l_j: the raw logit of each chosen expert ([hotelren]
// §3.2 skips the softmax).
int oracle_weights_for(const float* logits, int T, int E, int k, const int32_t* idx, int flags, float* w) {
  if (T < 0 || E <= 0 || k <= 0 || k > E) return ORC_EARG;
  if (flags & ~(ORC_ROUTER_CLAMP | ORC_ROUTER_RAW)) return ORC_EARG;
  for (int t = 0; t < T; ++t) {
    const float* l = logits + (int64_t)t * E;
    const int32_t* id = idx + (int64_t)t * k;
    double lmax = -INFINITY;
    for (int j = 0; j < k; ++j) {
      if (id[j] < 0 || id[j] >= E) return ORC_EARG;
      lmax = std::max(lmax, (double)l[id[j]]);
    }
    if (flags & ORC_ROUTER_RAW) {
      for (int j = 0; j < k; ++j) w[(int64_t)t * k + j] = l[id[j]];
      continue;
    }
    double den = 0.0;
    for (int j = 0; j < k; ++j) den += std::exp((double)l[id[j]] - lmax);
    for (int j = 0; j < k; ++j) w[(int64_t)t * k + j] = (float)(std::exp((double)l[id[j]] - lmax) / den);
  }
  return ORC_OK;
}

// Step 2, top-k: order the experts by (logit descending, index ascending) and keep the
// first k, slot 0 = largest.  The strict ">" of the per-token scan in [mhpq] §3.2 keeps the
// lower index on ties.  Also reports gap[t] = l_(k) - l_(k+1), the distance between the last
// chosen and the first unchosen logit (+inf when k == E), for the near-tie protocol.
int oracle_topk(const float* logits, int T, int E, int k, int flags, int32_t* idx, float* w, float* gap) {
  if (T < 0 || E <= 0 || k <= 0 || k > E) return ORC_EARG;
  std::vector<int> order(E);
  for (int t = 0; t < T; ++t) {
    const float* l = logits + (int64_t)t * E;
    for (int e = 0; e < E; ++e) order[e] = e;
    std::sort(order.begin(), order.end(), [l](int a, int b) {
      return l[a] > l[b] || (l[a] == l[b] && a < b);
    });
    for (int j = 0; j < k; ++j) idx[(int64_t)t * k + j] = order[j];
    if (gap) gap[t] = (k < E) ? (float)((double)l[order[k - 1]] - (double)l[order[k]]) : INFINITY;
  }
  return w ? oracle_weights_for(logits, T, E, k, idx, flags, w) : ORC_OK;
}

// Steps 4/5, counts, offsets and the permutation that groups rows by expert.
// counts[e] = #{(t, j) : idx[t][j] = e}; offsets[0] = 0, offsets[e+1] = offsets[e] + counts[e]
// ([pptc] §3.3 expert_offsets as a running sum of sizes).  Grouping ([trdm] §6.2: samples
// that activate the same expert are batched together) walks t ascending, then j ascending,
// and appends (t, j) to its expert's group: src_row[r] = t, dst_row[t][j] = r.
int oracle_group(const int32_t* idx, int T, int k, int E, int32_t* counts, int32_t* offsets,
                 int32_t* src_row, int32_t* dst_row) {
  if (T < 0 || k <= 0 || E <= 0) return ORC_EARG;
  for (int e = 0; e < E; ++e) counts[e] = 0;
  for (int64_t a = 0; a < (int64_t)T * k; ++a) {
    if (idx[a] < 0 || idx[a] >= E) return ORC_EARG;
    counts[idx[a]]++;
  }
  offsets[0] = 0;
  for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
  std::vector<int32_t> cursor(E, 0);
  for (int t = 0; t < T; ++t)
    for (int j = 0; j < k; ++j) {
      const int e = idx[(int64_t)t * k + j];
      const int32_t r = offsets[e] + cursor[e]++;
      src_row[r] = t;
      dst_row[(int64_t)t * k + j] = r;
    }
  return ORC_OK;
}

// Step 6 on one (token, expert) pair: Yp = W2_e (silu(W1_e x_t) * (W3_e x_t)).
// Experts live in one buffer at a fixed stride ([mhpq] §2.1: address = id * EXPERT_SIZE;
// [0539edu] §3.1: one expert's parameters contiguous): expert e starts at e * stride.
int oracle_expert_row(const void* x, int act, int d, int t, const void* expert_w, int wdt,
                      int64_t stride, int f, const float* scales, int e, float* yrow) {
  std::vector<double> xr(d);
  for (int i = 0; i < d; ++i) xr[i] = widen(x, act, (int64_t)t * d + i);
  if (quantised(wdt) && !scales) return ORC_EARG;
  if (wdt == ORC_I4 && (d % kI4Group || f % kI4Group)) return ORC_EARG;
  const float* sc = quantised(wdt) ? scales + (int64_t)e * expert_scale_count(wdt, d, f) : nullptr;
  return expert_ffn(xr.data(), d, f, expert_w, wdt, (int64_t)e * stride, sc, yrow) ? ORC_OK
                                                                                    : ORC_ENONFINITE;
}

// Step 7, combine for the tokens listed: y[t] = sum_{j=0..k-1} w[t][j] * FFN_{idx[t][j]}(x_t),
// summed in j order, plus the shared expert's FFN(x_t) with weight 1 when fs > 0.
// [hotelren] §2.1 step 6 and §2.3 combine_kernel (weighted sum of the k expert outputs),
// [pptc] §2.1 (k-way aggregation).
// y is [ntok, d] in the order of `tokens`.
int oracle_combine(const void* x, int act, int T, int d, int k, const int32_t* idx,
                   const float* w, const void* expert_w, int wdt, int64_t stride, int f,
                   const float* scales, const void* shared_w, int fs, const int32_t* tokens,
                   int ntok, float* y) {
  if (d <= 0 || k <= 0 || f <= 0 || ntok < 0) return ORC_EARG;
  if (quantised(wdt) && !scales) return ORC_EARG;
  if (wdt == ORC_I4 && (d % kI4Group || f % kI4Group)) return ORC_EARG;
  if (fs > 0 && (!shared_w || quantised(wdt))) return ORC_EARG;
  std::vector<float> yp(d), ys(d);
  std::vector<double> xr(d);
  for (int n = 0; n < ntok; ++n) {
    const int t = tokens[n];
    if (t < 0 || t >= T) return ORC_EARG;
    for (int i = 0; i < d; ++i) xr[i] = widen(x, act, (int64_t)t * d + i);
    std::vector<double> acc(d, 0.0);
    for (int j = 0; j < k; ++j) {
      const int e = idx[(int64_t)t * k + j];
      const float* sc = quantised(wdt) ? scales + (int64_t)e * expert_scale_count(wdt, d, f) : nullptr;
      if (!expert_ffn(xr.data(), d, f, expert_w, wdt, (int64_t)e * stride, sc, yp.data()))
        return ORC_ENONFINITE;
      const double wj = (double)w[(int64_t)t * k + j];
      for (int i = 0; i < d; ++i) acc[i] += wj * (double)yp[i];
    }
    if (fs > 0) {
      if (!expert_ffn(xr.data(), d, fs, shared_w, wdt, 0, nullptr, ys.data())) return ORC_ENONFINITE;
      for (int i = 0; i < d; ++i) acc[i] += (double)ys[i];
    }
    for (int i = 0; i < d; ++i) y[(int64_t)n * d + i] = (float)acc[i];
  }
  return ORC_OK;
}

// One dequantised weight element W[o][i] (as `weight` above) of the [rows, cols] matrix at
// element offset `base`, with that matrix's scales; exposed so that tests can pin the storage
// formats element by element.
int oracle_weight_element(const void* w, int wdt, int64_t base, int64_t rows, int64_t cols, int64_t o, int64_t i,
                          const float* scale, double* out) {
  if (!w || !out || rows <= 0 || cols <= 0 || o < 0 || o >= rows || i < 0 || i >= cols) return ORC_EARG;
  if (quantised(wdt) && !scale) return ORC_EARG;
  if (wdt == ORC_I4 && cols % kI4Group) return ORC_EARG;
  *out = weight(w, wdt, base, rows, cols, o, i, scale);
  return ORC_OK;
}

// The whole layer: steps 1-7 for every token.  Any output pointer may be NULL except y.
int oracle_moe_forward(const void* x, int act, int T, int d, const void* router_w,
                       const float* router_b, int E, int k, int flags, const void* expert_w, int wdt,
                       int64_t stride, int f, const float* scales, const void* shared_w, int fs,
                       float* logits_out, int32_t* idx_out, float* w_out, int32_t* counts,
                       int32_t* offsets, int32_t* src_row, int32_t* dst_row, float* y) {
  if (T < 0 || d <= 0 || E <= 0 || k <= 0 || k > E || f <= 0) return ORC_EARG;
  if (T == 0) return ORC_OK;
  if (!y) return ORC_EARG;
  std::vector<float> logits((size_t)T * E), wv((size_t)T * k);
  std::vector<int32_t> iv((size_t)T * k), cnt(E), off(E + 1), src((size_t)T * k), dst((size_t)T * k);
  int rc = oracle_router_logits(x, act, T, d, router_w, router_b, E, flags, logits.data());
  if (rc) return rc;
  rc = oracle_topk(logits.data(), T, E, k, flags, iv.data(), wv.data(), nullptr);
  if (rc) return rc;
  rc = oracle_group(iv.data(), T, k, E, cnt.data(), off.data(), src.data(), dst.data());
  if (rc) return rc;
  // Expert compute over the grouped rows, then gather in token order.
  std::vector<float> yp((size_t)T * k * d);
  for (int r = 0; r < T * k; ++r) {
    int e = 0;
    while (off[e + 1] <= r) ++e;
    rc = oracle_expert_row(x, act, d, src[r], expert_w, wdt, stride, f, scales, e,
                           yp.data() + (size_t)r * d);
    if (rc) return rc;
  }
  std::vector<double> xr(d);
  std::vector<float> ys(d);
  for (int t = 0; t < T; ++t) {
    std::vector<double> acc(d, 0.0);
    for (int j = 0; j < k; ++j) {
      const float* row = yp.data() + (size_t)dst[(size_t)t * k + j] * d;
      const double wj = (double)wv[(size_t)t * k + j];
      for (int i = 0; i < d; ++i) acc[i] += wj * (double)row[i];
    }
    if (fs > 0) {
      for (int i = 0; i < d; ++i) xr[i] = widen(x, act, (int64_t)t * d + i);
      if (!expert_ffn(xr.data(), d, fs, shared_w, wdt, 0, nullptr, ys.data())) return ORC_ENONFINITE;
      for (int i = 0; i < d; ++i) acc[i] += (double)ys[i];
    }
    for (int i = 0; i < d; ++i) y[(size_t)t * d + i] = (float)acc[i];
  }
  if (logits_out) std::memcpy(logits_out, logits.data(), logits.size() * 4);
  if (idx_out) std::memcpy(idx_out, iv.data(), iv.size() * 4);
  if (w_out) std::memcpy(w_out, wv.data(), wv.size() * 4);
  if (counts) std::memcpy(counts, cnt.data(), cnt.size() * 4);
  if (offsets) std::memcpy(offsets, off.data(), off.size() * 4);
  if (src_row) std::memcpy(src_row, src.data(), src.size() * 4);
  if (dst_row) std::memcpy(dst_row, dst.data(), dst.size() * 4);
  return ORC_OK;
}

}  // extern "C"
