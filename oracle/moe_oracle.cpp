// Plain CPU oracle for the deterministic MoE layer, forward and backward.
//
// TEST INFRASTRUCTURE ONLY. Nothing on the product path may call, link or load
// this file: only the test suite, the package's smoke check and the benchmark's
// CPU-baseline leg use it. It shares no code, header, table or helper with the
// CUDA library; both sides are fed by the seeded input generators alone.
//
// Every function computes its step's plain definition, in the order the source
// pages state it, with no blocking, fusion or reordering beyond that. Floating
// point is fp64 except where the method fixes a narrower type (bf16 operands
// and bf16 rounding of the SwiGLU output, which is the second GEMM's operand;
// fp32 gates; the fp32 fixed-order combine, which is a definition in itself).
//
// Sources (page title, section):
//  [MoK-2]  "Mixture-of-Kittens: A MoE Megakernel for GB300 NVL72",
//           section 2 "Push vs. Pull", on-device schedule generation box:
//           counts T, M, offsets S, stable cross-rank position p, table Phi.
//  [MoK-3]  same page, section 3 "The Goldilocks Minibatch Size T": wave floor.
//  [MoK-5]  same page, section 5 "Megakernel Fusion": SwiGLU expert FFN.
//  [SCAN]   "Scan once, scatter once", section "The fix is a counting sort":
//           the four scheduler stages, 1,024 logical threads per peer,
//           2*P*R route reads, E*1024 counters, 256-row expert padding.
//  [BEYOND] "Beyond Peak TFLOPs", section 2.A (pull dispatch, two-column
//           table) and the MoK overview (fixed floating-point order).
//
// Readings where the pages are silent or garbled (each is also argued in the
// design notes):
//  R1 within one (expert, peer) pair, routes keep ascending route index
//     q = token*k + slot (the pages' thread-major order with contiguous
//     per-thread chunks);
//  R2 the placement formula's first sum runs over all peers and o is the
//     route's stable rank within its (expert, peer) pair;
//  R3 an expert with no routes gets 0 rows (0 is a multiple of 256);
//  R4 pad rows of Phi hold (-1,-1) and pad rows of the gathered buffer are 0;
//  R6 top-k ties go to the lower expert id; slots are in descending logit order;
//  R7 gates are the softmax over the chosen k logits, stored as fp32;
//  R8 SwiGLU: h = bf16_rne(silu(x.W1) * (x.W3)), y = h.W2;
//  R9 combine: out = bf16_rne(sum_j g_j * y_j) accumulated from 0 in
//     ascending slot order (the fp32 fixed-order form uses fmaf).
//  MX MXFP8 routed experts ("Mixture-of-Kittens", section 5; the OCP
//     Microscaling (MX) formats, MXFP8 with E4M3 elements): every GEMM operand
//     quantised in blocks of 32 along its reduction dimension, one E8M0 scale
//     per block (see the MX functions below).
//  B1 backward ("Mixture-of-Kittens", MoK overview: one table serves the
//     forward and backward phases; pull-reverse-combine, push-reverse-
//     dispatch; section 5: router gradients from the inner product of the
//     SwiGLU activations and the down-projection dgrads): the exact gradient
//     of the layer above, with bf16 rounding at every GEMM operand that is
//     not an input: the saved pre-activations a, b, the SwiGLU output h, the
//     SwiGLU input gradients da, db and the gate-scaled activations g*h.
#include <algorithm>
#include <cfenv>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

#ifdef _OPENMP
#include <omp.h>
#endif

namespace {

double bf16_to_double(uint16_t b) {
  uint32_t u = static_cast<uint32_t>(b) << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return static_cast<double>(f);
}

// Round a double to the nearest bf16 value, ties to even, straight from
// double (no intermediate fp32 rounding). bf16 keeps 8 significant bits and
// fp32's exponent range; its smallest subnormal is 2^-133.
uint16_t double_to_bf16(double v) {
  if (std::isnan(v)) return 0x7FC0;
  if (std::isinf(v)) return v > 0 ? 0x7F80 : 0xFF80;
  if (v == 0.0) return std::signbit(v) ? 0x8000 : 0x0000;
  int e;
  std::frexp(v, &e);                 // v = m * 2^e, 0.5 <= |m| < 1
  int q = std::max(e - 8, -133);     // weight of the last kept bit
  double scaled = std::ldexp(v, -q);
  double r = std::nearbyint(scaled); // default rounding mode: ties to even
  double rv = std::ldexp(r, q);
  float f = static_cast<float>(rv);  // exact unless it overflows to inf
  uint32_t u;
  std::memcpy(&u, &f, 4);
  return static_cast<uint16_t>(u >> 16);
}

}  // namespace

extern "C" {

int oracle_num_threads() {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

void oracle_set_num_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

// bf16 rounding exposed for the oracle's own pins.
uint16_t oracle_round_bf16(double v) { return double_to_bf16(v); }

// ---------------------------------------------------------------------------
// Step 1: top-k routing and gates (R6, R7).
// For each token: order experts by (logit descending, id ascending), keep the
// first k as slots 0..k-1; g_j = exp(l_j - l_0) / sum_j' exp(l_j' - l_0),
// i.e. the softmax restricted to the chosen logits.
// ---------------------------------------------------------------------------
int oracle_route_topk(const float* logits, int64_t n_tokens, int32_t E, int32_t k,
                      int32_t* ids, float* gates32, double* gates64) {
  if (E <= 0 || k <= 0 || k > E || n_tokens < 0) return 1;
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < n_tokens; ++t) {
    const float* row = logits + t * E;
    std::vector<int32_t> order(E);
    for (int32_t e = 0; e < E; ++e) order[e] = e;
    std::sort(order.begin(), order.end(), [row](int32_t a, int32_t b) {
      if (row[a] != row[b]) return row[a] > row[b];
      return a < b;
    });
    double l0 = row[order[0]];
    double denom = 0.0;
    for (int32_t j = 0; j < k; ++j) denom += std::exp(static_cast<double>(row[order[j]]) - l0);
    for (int32_t j = 0; j < k; ++j) {
      double g = std::exp(static_cast<double>(row[order[j]]) - l0) / denom;
      ids[t * k + j] = order[j];
      if (gates64) gates64[t * k + j] = g;
      if (gates32) gates32[t * k + j] = static_cast<float>(g);
    }
  }
  return 0;
}

// ---------------------------------------------------------------------------
// Step 2: the pull-dispatch schedule Phi as a counting sort [SCAN], with the
// stable cross-peer position of [MoK-2].
//
// ids: [P, N, k] expert ids. Route (r, q) is token i = q / k, slot j = q % k of
// peer r; R = N*k routes per peer. Each peer's routes are split among 1,024
// logical scheduler threads, thread t owning the contiguous chunk
// [t*ceil(R/1024), (t+1)*ceil(R/1024)) (R1).
//   stage 1  count routes per (expert l, peer r, thread t)
//   stage 2  prefix the per-thread counts: base[l][r][t] = sum_{t'<t} cnt
//   stage 3  M[l][r] = sum_t cnt; T[l] = sum_r M[l][r];
//            Tp[l] = ceil(T[l]/pad)*pad; S = exclusive prefix sum of Tp
//   stage 4  scatter every route once: o = base + running count in its
//            thread; p = sum_{r'} min(M[l][r'], o) + |{r' < r : M[l][r'] > o}|;
//            Phi[S[l]+p] = (r, i); route_row[r][q] = S[l] + p
// Rows S[l]+T[l] .. S[l+1]-1 are padding, Phi = (-1,-1) (R4).
//
// Outputs: phi [rows_cap, 2], offsets [E+1] (= S, with S[E] = total rows),
// counts [E, P] (= M), route_row [P, N, k].
// stats[0] = route reads performed (each route is read by stage 1 and stage 4),
// stats[1] = counter words used (E * P * 1024), stats[2] = logical threads/peer.
// Returns 0, or 1 on bad arguments, 2 if an id is outside [0, E), 3 if
// rows_cap is too small.
// ---------------------------------------------------------------------------
int oracle_schedule(const int32_t* ids, int32_t P, int32_t N, int32_t k, int32_t E, int32_t pad,
                    int64_t rows_cap, int32_t* phi, int32_t* offsets, int32_t* counts,
                    int32_t* route_row, int64_t* stats) {
  if (P <= 0 || N < 0 || k <= 0 || E <= 0 || pad <= 0) return 1;
  const int64_t R = static_cast<int64_t>(N) * k;
  const int64_t THREADS = 1024;
  const int64_t chunk = (R + THREADS - 1) / THREADS;
  int64_t reads = 0;

  // stage 1: count per (expert, peer, logical thread)
  std::vector<int64_t> cnt(static_cast<size_t>(E) * P * THREADS, 0);
  auto C = [&](int64_t l, int64_t r, int64_t t) -> int64_t& { return cnt[(l * P + r) * THREADS + t]; };
  for (int64_t r = 0; r < P; ++r) {
    for (int64_t q = 0; q < R; ++q) {
      int32_t l = ids[r * R + q];
      ++reads;
      if (l < 0 || l >= E) return 2;
      C(l, r, q / chunk) += 1;
    }
  }
  // stage 2: thread-major prefix within each (expert, peer)
  std::vector<int64_t> base(cnt.size(), 0);
  std::vector<int64_t> M(static_cast<size_t>(E) * P, 0);
  for (int64_t l = 0; l < E; ++l)
    for (int64_t r = 0; r < P; ++r) {
      int64_t run = 0;
      for (int64_t t = 0; t < THREADS; ++t) {
        base[(l * P + r) * THREADS + t] = run;
        run += C(l, r, t);
      }
      M[l * P + r] = run;
    }
  // stage 3: totals, padding, segment bases
  std::vector<int64_t> S(E + 1, 0), Tl(E, 0);
  for (int64_t l = 0; l < E; ++l) {
    int64_t T = 0;
    for (int64_t r = 0; r < P; ++r) T += M[l * P + r];
    Tl[l] = T;
    int64_t Tp = (T + pad - 1) / pad * pad;
    S[l + 1] = S[l] + Tp;
  }
  if (S[E] > rows_cap) return 3;
  if (S[E] > INT32_MAX) return 1;
  for (int64_t l = 0; l <= E; ++l) offsets[l] = static_cast<int32_t>(S[l]);
  for (int64_t l = 0; l < E; ++l)
    for (int64_t r = 0; r < P; ++r) counts[l * P + r] = static_cast<int32_t>(M[l * P + r]);
  for (int64_t l = 0; l < E; ++l)
    for (int64_t row = S[l] + Tl[l]; row < S[l + 1]; ++row) {
      phi[2 * row] = -1;
      phi[2 * row + 1] = -1;
    }
  // stage 4: scatter each route once
  std::vector<int64_t> running(static_cast<size_t>(E) * THREADS, 0);
  for (int64_t r = 0; r < P; ++r) {
    std::fill(running.begin(), running.end(), 0);
    for (int64_t q = 0; q < R; ++q) {
      int32_t l = ids[r * R + q];
      ++reads;
      int64_t t = q / chunk;
      int64_t o = base[(l * P + r) * THREADS + t] + running[l * THREADS + t];
      running[l * THREADS + t] += 1;
      int64_t p = 0;
      for (int64_t r2 = 0; r2 < P; ++r2) p += std::min(M[l * P + r2], o);
      for (int64_t r2 = 0; r2 < r; ++r2) p += (M[l * P + r2] > o) ? 1 : 0;
      int64_t row = S[l] + p;
      phi[2 * row] = static_cast<int32_t>(r);
      phi[2 * row + 1] = static_cast<int32_t>(q / k);
      route_row[r * R + q] = static_cast<int32_t>(row);
    }
  }
  if (stats) {
    stats[0] = reads;
    stats[1] = static_cast<int64_t>(E) * P * THREADS;
    stats[2] = THREADS;
  }
  return 0;
}

// Placement by the closed form alone: o is found by a plain sequential scan of
// the peer's routes (no per-thread counting), then p by the [MoK-2] formula.
// Fills route_row [P, N, k] and offsets [E+1]. Returns 0, 1 or 2 as above.
int oracle_place_closed_form(const int32_t* ids, int32_t P, int32_t N, int32_t k, int32_t E,
                             int32_t pad, int32_t* offsets, int32_t* route_row) {
  if (P <= 0 || N < 0 || k <= 0 || E <= 0 || pad <= 0) return 1;
  const int64_t R = static_cast<int64_t>(N) * k;
  std::vector<int64_t> M(static_cast<size_t>(E) * P, 0);
  for (int64_t r = 0; r < P; ++r)
    for (int64_t q = 0; q < R; ++q) {
      int32_t l = ids[r * R + q];
      if (l < 0 || l >= E) return 2;
      M[l * P + r] += 1;
    }
  std::vector<int64_t> S(E + 1, 0);
  for (int64_t l = 0; l < E; ++l) {
    int64_t T = 0;
    for (int64_t r = 0; r < P; ++r) T += M[l * P + r];
    S[l + 1] = S[l] + (T + pad - 1) / pad * pad;
  }
  for (int64_t l = 0; l <= E; ++l) offsets[l] = static_cast<int32_t>(S[l]);
  std::vector<int64_t> seen(E, 0);
  for (int64_t r = 0; r < P; ++r) {
    std::fill(seen.begin(), seen.end(), 0);
    for (int64_t q = 0; q < R; ++q) {
      int32_t l = ids[r * R + q];
      int64_t o = seen[l]++;
      int64_t p = 0;
      for (int64_t r2 = 0; r2 < P; ++r2) p += std::min(M[l * P + r2], o);
      for (int64_t r2 = 0; r2 < r; ++r2) p += (M[l * P + r2] > o) ? 1 : 0;
      route_row[r * R + q] = static_cast<int32_t>(S[l] + p);
    }
  }
  return 0;
}

// Placement by explicit simulation of the round-robin: for each expert, one
// FIFO per peer holds that peer's routes in ascending q; rows are handed out
// by visiting peers 0..P-1 in turn, popping one route from each non-empty
// FIFO, until all are empty; then the segment is padded to a multiple of pad.
// Fills route_row, offsets and phi (rows_cap rows). Returns 0, 1, 2 or 3.
int oracle_place_queue_sim(const int32_t* ids, int32_t P, int32_t N, int32_t k, int32_t E,
                           int32_t pad, int64_t rows_cap, int32_t* offsets, int32_t* route_row,
                           int32_t* phi) {
  if (P <= 0 || N < 0 || k <= 0 || E <= 0 || pad <= 0) return 1;
  const int64_t R = static_cast<int64_t>(N) * k;
  std::vector<std::vector<std::vector<int64_t>>> fifo(E, std::vector<std::vector<int64_t>>(P));
  for (int64_t r = 0; r < P; ++r)
    for (int64_t q = 0; q < R; ++q) {
      int32_t l = ids[r * R + q];
      if (l < 0 || l >= E) return 2;
      fifo[l][r].push_back(q);
    }
  int64_t row = 0;
  for (int64_t l = 0; l < E; ++l) {
    offsets[l] = static_cast<int32_t>(row);
    std::vector<size_t> head(P, 0);
    bool any = true;
    while (any) {
      any = false;
      for (int64_t r = 0; r < P; ++r) {
        if (head[r] < fifo[l][r].size()) {
          int64_t q = fifo[l][r][head[r]++];
          if (row >= rows_cap) return 3;
          route_row[r * R + q] = static_cast<int32_t>(row);
          phi[2 * row] = static_cast<int32_t>(r);
          phi[2 * row + 1] = static_cast<int32_t>(q / k);
          ++row;
          any = true;
        }
      }
    }
    while ((row - offsets[l]) % pad != 0) {
      if (row >= rows_cap) return 3;
      phi[2 * row] = -1;
      phi[2 * row + 1] = -1;
      ++row;
    }
  }
  offsets[E] = static_cast<int32_t>(row);
  return 0;
}

// Wave floor of [MoK-3]: the smallest T with T*min(2I, H) >= 2C*128*256, i.e.
// enough 128x256 output tiles for two waves over C SMs in both the up/gate and
// the down projection. Returns ceil(2C*128*256 / min(2I, H)).
int64_t oracle_wave_floor(int64_t H, int64_t I, int64_t C) {
  int64_t d = std::min(2 * I, H);
  if (d <= 0) return -1;
  int64_t num = 2 * C * 128 * 256;
  return (num + d - 1) / d;
}

// ---------------------------------------------------------------------------
// Step 3: pull dispatch [BEYOND 2.A]: the destination row is a copy of token
// (src_rank, src_idx) = Phi[row]; padding rows are zero (R4).
// x: [P*N, H] bf16 bits; rows: the n row indices of Phi to gather; xg: [n, H].
// ---------------------------------------------------------------------------
void oracle_dispatch_rows(const uint16_t* x, int32_t N, int32_t H, const int32_t* phi,
                          const int64_t* rows, int64_t n, uint16_t* xg) {
#pragma omp parallel for schedule(static)
  for (int64_t a = 0; a < n; ++a) {
    int64_t row = rows[a];
    int32_t src_rank = phi[2 * row], src_idx = phi[2 * row + 1];
    uint16_t* dst = xg + a * H;
    if (src_rank < 0) {
      std::memset(dst, 0, sizeof(uint16_t) * H);
    } else {
      const uint16_t* src = x + (static_cast<int64_t>(src_rank) * N + src_idx) * H;
      std::memcpy(dst, src, sizeof(uint16_t) * H);
    }
  }
}

// ---------------------------------------------------------------------------
// Step 4: grouped SwiGLU expert FFN [MoK-5], one row at a time (R8).
// xg: [n, H] rows, expert[a] the expert of row a; W1[e], W3[e] point to that
// expert's [H, I] matrices, W2[e] to its [I, H] matrix (bf16 bits, row-major).
// a = x.W1, b = x.W3 in fp64; h = bf16_rne(a / (1 + exp(-a)) * b);
// y = h.W2 in fp64. Outputs h [n, I] (bf16 bits) and y [n, H] (fp64).
// ---------------------------------------------------------------------------
void oracle_ffn_rows(const uint16_t* xg, int64_t n, const int32_t* expert, int32_t H, int32_t I,
                     const uint16_t* const* W1, const uint16_t* const* W3,
                     const uint16_t* const* W2, uint16_t* h, double* y) {
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t a = 0; a < n; ++a) {
    const int32_t e = expert[a];
    const uint16_t* xr = xg + a * H;
    const uint16_t* w1 = W1[e];
    const uint16_t* w3 = W3[e];
    const uint16_t* w2 = W2[e];
    std::vector<double> acc_a(I, 0.0), acc_b(I, 0.0), hv(I, 0.0);
    for (int32_t c = 0; c < H; ++c) {
      const double xv = bf16_to_double(xr[c]);
      const uint16_t* w1r = w1 + static_cast<int64_t>(c) * I;
      const uint16_t* w3r = w3 + static_cast<int64_t>(c) * I;
      for (int32_t i = 0; i < I; ++i) {
        acc_a[i] += xv * bf16_to_double(w1r[i]);
        acc_b[i] += xv * bf16_to_double(w3r[i]);
      }
    }
    for (int32_t i = 0; i < I; ++i) {
      const double s = acc_a[i] / (1.0 + std::exp(-acc_a[i]));
      const uint16_t hb = double_to_bf16(s * acc_b[i]);
      h[a * I + i] = hb;
      hv[i] = bf16_to_double(hb);
    }
    double* yr = y + a * H;
    for (int32_t c = 0; c < H; ++c) yr[c] = 0.0;
    for (int32_t i = 0; i < I; ++i) {
      const double v = hv[i];
      const uint16_t* w2r = w2 + static_cast<int64_t>(i) * H;
      for (int32_t c = 0; c < H; ++c) yr[c] += v * bf16_to_double(w2r[c]);
    }
  }
}

// ---------------------------------------------------------------------------
// Step 5: push combine in a fixed floating-point order [BEYOND], (R9).
// For token a (n tokens), slot j: its expert output is row sel[a*k + j] of y
// ([y_rows, H]); out[a] = sum_j g[a*k+j] * y[sel[a*k+j]].
// oracle_combine_f64: fp64 sum in ascending j; writes the unrounded result
// (out64, may be null) and its bf16 rounding (out_bf16, may be null).
// oracle_combine_f32: the fixed-order fp32 form: acc = 0.0f, then
// acc = fmaf(g_j, y_j, acc) for j = 0..k-1, then one bf16 rounding.
// A slot whose sel is negative contributes nothing.
// ---------------------------------------------------------------------------
void oracle_combine_f64(const double* y, int32_t H, const int64_t* sel, const double* g, int64_t n,
                        int32_t k, double* out64, uint16_t* out_bf16) {
#pragma omp parallel for schedule(static)
  for (int64_t a = 0; a < n; ++a) {
    for (int32_t c = 0; c < H; ++c) {
      double acc = 0.0;
      for (int32_t j = 0; j < k; ++j) {
        const int64_t s = sel[a * k + j];
        if (s < 0) continue;
        acc += g[a * k + j] * y[s * H + c];
      }
      if (out64) out64[a * H + c] = acc;
      if (out_bf16) out_bf16[a * H + c] = double_to_bf16(acc);
    }
  }
}

void oracle_combine_f32(const float* y, int32_t H, const int64_t* sel, const float* g, int64_t n,
                        int32_t k, uint16_t* out_bf16) {
#pragma omp parallel for schedule(static)
  for (int64_t a = 0; a < n; ++a) {
    for (int32_t c = 0; c < H; ++c) {
      float acc = 0.0f;
      for (int32_t j = 0; j < k; ++j) {
        const int64_t s = sel[a * k + j];
        if (s < 0) continue;
        acc = std::fmaf(g[a * k + j], y[s * H + c], acc);
      }
      out_bf16[a * H + c] = double_to_bf16(static_cast<double>(acc));
    }
  }
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Backward (B1). For one route row with token activations x (the gathered
// row), upstream gradient d (the token's dout row), gate g and expert e:
//   a = x.W1[e], b = x.W3[e]                 (fp64)
//   h = silu(a) * b                          (rounded to bf16: the forward's h)
//   as, bs = a, b                            (rounded to bf16: saved activations)
//   dhu = d . W2[e]^T                        dhu[i] = sum_c d[c] W2[e][i][c]
//   dgate = sum_i h[i] dhu[i]                (the gate's gradient, SonicMoE form)
//   dh = g * dhu
//   s = 1 / (1 + exp(-as))
//   da = dh * bs * s * (1 + as * (1 - s))    (d silu(a)/da = s (1 + a (1 - s)))
//   db = dh * as * s                         (rounded to bf16: GEMM operands)
//   hg = g * h                               (rounded to bf16: the dW2 operand)
//   dx_row = da . W1[e]^T + db . W3[e]^T     dx_row[c] = sum_i da[i] W1[e][c][i] + db[i] W3[e][c][i]
// exact != 0 drops every bf16 rounding: the plain real-number gradient.
// ---------------------------------------------------------------------------
namespace {

// The rounded mode rounds each bf16 operand once, from its exact value.
double rnd(double v, int exact) { return exact ? v : bf16_to_double(double_to_bf16(v)); }

// The element-wise part for one (row, column i): from a, b (unrounded), dhu
// and g, the values the two backward GEMMs and the gate gradient consume.
struct BwdElem {
  double h, da, db, hg;
};

BwdElem swiglu_bwd_elem(double a, double b, double dhu, double g, int exact) {
  BwdElem r;
  r.h = rnd(a / (1.0 + std::exp(-a)) * b, exact);
  const double as = rnd(a, exact), bs = rnd(b, exact);
  const double dh = g * dhu;
  const double s = 1.0 / (1.0 + std::exp(-as));
  r.da = rnd(dh * bs * s * (1.0 + as * (1.0 - s)), exact);
  r.db = rnd(dh * as * s, exact);
  r.hg = rnd(g * r.h, exact);
  return r;
}

}  // namespace

extern "C" {

// Per-row backward through the expert FFN (B1).
// xg, dys: [n, H] bf16 bits (the row's token activations and its token's
// upstream gradient); g: [n] gate of the row's route; expert: [n].
// Outputs (each may be null): dgate [n] fp64; dxg [n, H] fp64;
// da, db, hg [n, I] (exact == 0: bf16 bits of the rounded values; ignored
// when exact != 0).
void oracle_ffn_bwd_rows(const uint16_t* xg, const uint16_t* dys, const double* g, int64_t n,
                         const int32_t* expert, int32_t H, int32_t I,
                         const uint16_t* const* W1, const uint16_t* const* W3,
                         const uint16_t* const* W2, int exact, double* dgate, double* dxg,
                         uint16_t* da_out, uint16_t* db_out, uint16_t* hg_out) {
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t r = 0; r < n; ++r) {
    const int32_t e = expert[r];
    const uint16_t* xr = xg + r * H;
    const uint16_t* dr = dys + r * H;
    const uint16_t* w1 = W1[e];
    const uint16_t* w3 = W3[e];
    const uint16_t* w2 = W2[e];
    std::vector<double> a(I, 0.0), b(I, 0.0), dhu(I, 0.0), da(I), db(I);
    for (int32_t c = 0; c < H; ++c) {
      const double xv = bf16_to_double(xr[c]);
      for (int32_t i = 0; i < I; ++i) {
        a[i] += xv * bf16_to_double(w1[static_cast<int64_t>(c) * I + i]);
        b[i] += xv * bf16_to_double(w3[static_cast<int64_t>(c) * I + i]);
      }
    }
    for (int32_t i = 0; i < I; ++i) {
      double acc = 0.0;
      for (int32_t c = 0; c < H; ++c)
        acc += bf16_to_double(dr[c]) * bf16_to_double(w2[static_cast<int64_t>(i) * H + c]);
      dhu[i] = acc;
    }
    double dg = 0.0;
    for (int32_t i = 0; i < I; ++i) {
      const BwdElem v = swiglu_bwd_elem(a[i], b[i], dhu[i], g[r], exact);
      dg += v.h * dhu[i];
      da[i] = v.da;
      db[i] = v.db;
      if (!exact) {
        if (da_out) da_out[r * I + i] = double_to_bf16(v.da);
        if (db_out) db_out[r * I + i] = double_to_bf16(v.db);
        if (hg_out) hg_out[r * I + i] = double_to_bf16(v.hg);
      }
    }
    if (dgate) dgate[r] = dg;
    if (dxg) {
      for (int32_t c = 0; c < H; ++c) {
        double acc = 0.0;
        for (int32_t i = 0; i < I; ++i)
          acc += da[i] * bf16_to_double(w1[static_cast<int64_t>(c) * I + i]) +
                 db[i] * bf16_to_double(w3[static_cast<int64_t>(c) * I + i]);
        dxg[r * H + c] = acc;
      }
    }
  }
}

// Weight gradients of one expert (B1), accumulated over all R rows the
// expert received ("in one pass over the token dimension"):
//   dW1[c][i] = sum_rows x[c] da[i],  dW3[c][i] = sum_rows x[c] db[i],
//   dW2[i][c] = sum_rows hg[i] d[c].
// Only the entries at the chosen columns are formed: hs (n_h values of c)
// and is (n_i values of i); outputs dW1s, dW3s [n_h, n_i], dW2s [n_i, n_h].
// xg, dys: [R, H] bf16 bits; g: [R].
void oracle_wgrad_expert(const uint16_t* xg, const uint16_t* dys, const double* g, int64_t R,
                         int32_t H, int32_t I, const uint16_t* W1e, const uint16_t* W3e,
                         const uint16_t* W2e, const int32_t* hs, int32_t n_h, const int32_t* is,
                         int32_t n_i, int exact, double* dW1s, double* dW3s, double* dW2s) {
#pragma omp parallel for schedule(dynamic, 1)
  for (int32_t q = 0; q < n_i; ++q) {
    const int32_t i = is[q];
    std::vector<double> da(R), db(R), hg(R);
    for (int64_t r = 0; r < R; ++r) {
      double a = 0.0, b = 0.0, dhu = 0.0;
      for (int32_t c = 0; c < H; ++c) {
        const double xv = bf16_to_double(xg[r * H + c]);
        a += xv * bf16_to_double(W1e[static_cast<int64_t>(c) * I + i]);
        b += xv * bf16_to_double(W3e[static_cast<int64_t>(c) * I + i]);
        dhu += bf16_to_double(dys[r * H + c]) * bf16_to_double(W2e[static_cast<int64_t>(i) * H + c]);
      }
      const BwdElem v = swiglu_bwd_elem(a, b, dhu, g[r], exact);
      da[r] = v.da;
      db[r] = v.db;
      hg[r] = v.hg;
    }
    for (int32_t p = 0; p < n_h; ++p) {
      const int32_t c = hs[p];
      double s1 = 0.0, s3 = 0.0, s2 = 0.0;
      for (int64_t r = 0; r < R; ++r) {
        const double xv = bf16_to_double(xg[r * H + c]);
        s1 += xv * da[r];
        s3 += xv * db[r];
        s2 += hg[r] * bf16_to_double(dys[r * H + c]);
      }
      dW1s[static_cast<int64_t>(p) * n_i + q] = s1;
      dW3s[static_cast<int64_t>(p) * n_i + q] = s3;
      dW2s[static_cast<int64_t>(q) * n_h + p] = s2;
    }
  }
}

// Router backward (B1): gates g_j = softmax over the chosen logits l_j, so
// dL/dl_j = g_j (dgate_j - sum_j' g_j' dgate_j'); logits that were not
// chosen get 0. dgate, g, ids: [n, k]; dlogits: [n, E] (fp64).
void oracle_router_bwd(const double* dgate, const double* g, const int32_t* ids, int64_t n,
                       int32_t k, int32_t E, double* dlogits) {
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < n; ++t) {
    double* out = dlogits + t * E;
    for (int32_t e = 0; e < E; ++e) out[e] = 0.0;
    double s = 0.0;
    for (int32_t j = 0; j < k; ++j) s += g[t * k + j] * dgate[t * k + j];
    for (int32_t j = 0; j < k; ++j) out[ids[t * k + j]] = g[t * k + j] * (dgate[t * k + j] - s);
  }
}

}  // extern "C"

// ---------------------------------------------------------------------------
// MXFP8 (MX). E4M3 element: 1 sign bit, 4 exponent bits (bias 7), 3 mantissa
// bits; no infinities; S.1111.111 is NaN; the largest finite magnitude is
// 448 = 1.75 * 2^8; below 2^-6 the values are subnormal with step 2^-9. The
// code of a non-negative finite value is monotonic in the value. E8M0 scale:
// X = 2^(code - 127). For each block of 32 consecutive values along the
// reduction dimension:
//   amax = max |v_i|;  e = floor(log2 amax) - 8, clamped to [-127, 127]
//   (8: the exponent of E4M3's largest normal); an all-zero block takes -127;
//   q_i = E4M3(v_i / 2^e): nearest, ties to even; magnitudes above 448
//   clamp to 448 (the only finite choice: 480 would be the NaN code).
// ---------------------------------------------------------------------------
namespace {

double e4m3_value(uint8_t c) {
  const int E = (c >> 3) & 15, M = c & 7;
  if (E == 15 && M == 7) return std::nan("");
  const double mag = E == 0 ? std::ldexp(static_cast<double>(M), -9)
                            : std::ldexp(static_cast<double>(8 + M), E - 10);
  return (c & 0x80) ? -mag : mag;
}

uint8_t e4m3_encode(double v) {
  const uint8_t sign = std::signbit(v) ? 0x80 : 0x00;
  if (std::isnan(v)) return sign | 0x7F;
  const double a = std::fabs(v);
  if (!(a < 464.0)) return sign | 0x7E;   // 448: saturate (ties at 464 go to even 448)
  if (a < std::ldexp(1.0, -6)) {          // subnormal: code = value / 2^-9 (0..8, 8 = 2^-6)
    const double m = std::nearbyint(std::ldexp(a, 9));
    return sign | static_cast<uint8_t>(m);
  }
  int x;
  std::frexp(a, &x);                      // a = f * 2^x, 0.5 <= f < 1: floor(log2 a) = x - 1
  const int e = x - 1;
  double m = std::nearbyint(std::ldexp(a, 3 - e));  // 8..16 units of 2^(e-3)
  int ee = e;
  if (m == 16.0) {
    m = 8.0;
    ++ee;
  }
  int code = ((ee + 7) << 3) | (static_cast<int>(m) - 8);
  if (code > 0x7E) code = 0x7E;
  return sign | static_cast<uint8_t>(code);
}

}  // namespace

extern "C" {

double oracle_e4m3_value(uint8_t c) { return e4m3_value(c); }
uint8_t oracle_e4m3_encode(double v) { return e4m3_encode(v); }

// MX quantisation of n rows of K values (K a multiple of 32), blocks along
// the row: q [n, K] E4M3 codes, scale [n, K/32] E8M0 codes.
void oracle_mx_quantize(const double* v, int64_t n, int32_t K, uint8_t* q, uint8_t* scale) {
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < n; ++r) {
    for (int32_t b = 0; b < K / 32; ++b) {
      const double* blk = v + r * K + b * 32;
      double amax = 0.0;
      for (int i = 0; i < 32; ++i) amax = std::max(amax, std::fabs(blk[i]));
      int e = -127;
      if (amax > 0.0) {
        int x;
        std::frexp(amax, &x);
        e = std::min(127, std::max(-127, x - 1 - 8));
      }
      scale[r * (K / 32) + b] = static_cast<uint8_t>(e + 127);
      for (int i = 0; i < 32; ++i) q[r * K + b * 32 + i] = e4m3_encode(std::ldexp(blk[i], -e));
    }
  }
}

// The values the quantised rows stand for: q * 2^(scale - 127).
void oracle_mx_dequantize(const uint8_t* q, const uint8_t* scale, int64_t n, int32_t K,
                          double* out) {
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < n; ++r)
    for (int32_t i = 0; i < K; ++i)
      out[r * K + i] = std::ldexp(e4m3_value(q[r * K + i]), scale[r * (K / 32) + i / 32] - 127);
}

}  // extern "C"

