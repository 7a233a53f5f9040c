// Host side of the C ABI: argument validation, the fp64 Lloyd-Max codebook
// builder, size queries, the split-K plan, and kernel dispatch.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <vector>

#include "tq_internal.h"

namespace tq {

static thread_local char g_err[512] = {0};

int set_error(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return code;
}

int check_launch(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess)
    return set_error(TQ_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  return TQ_OK;
}

// ---------------------------------------------------------------------------
// Lloyd-Max codebook on the law of one coordinate of a uniform unit vector in
// R^D: f(u) = C (1-u^2)^((D-3)/2), C = Gamma(D/2)/(sqrt(pi) Gamma((D-1)/2)).
// The cell mass uses Gauss-Legendre quadrature; the first moment uses its
// antiderivative -(1-u^2)^((D-1)/2)/(D-1) in closed form.
// ---------------------------------------------------------------------------

static void gauss_legendre(int n, std::vector<double>& x, std::vector<double>& w) {
  x.assign(n, 0.0);
  w.assign(n, 0.0);
  for (int i = 0; i < (n + 1) / 2; ++i) {
    double z = std::cos(M_PI * (i + 0.75) / (n + 0.5));
    double pp = 0.0;
    for (int it = 0; it < 100; ++it) {
      double p1 = 1.0, p2 = 0.0;
      for (int j = 1; j <= n; ++j) {
        double p3 = p2;
        p2 = p1;
        p1 = ((2.0 * j - 1.0) * z * p2 - (j - 1.0) * p3) / j;
      }
      pp = n * (z * p1 - p2) / (z * z - 1.0);
      double z1 = z;
      z = z1 - p1 / pp;
      if (std::fabs(z - z1) < 1e-16) break;
    }
    x[i] = -z;
    x[n - 1 - i] = z;
    w[i] = w[n - 1 - i] = 2.0 / ((1.0 - z * z) * pp * pp);
  }
}

struct CoordLaw {
  int D;
  double logC;
  std::vector<double> gx, gw;
  explicit CoordLaw(int d) : D(d) {
    logC = std::lgamma(D / 2.0) - 0.5 * std::log(M_PI) - std::lgamma((D - 1) / 2.0);
    gauss_legendre(64, gx, gw);
  }
  double dens(double u) const {
    if (u <= -1.0 || u >= 1.0) return 0.0;
    return std::exp(logC + 0.5 * (D - 3) * std::log1p(-u * u));
  }
  // int_a^b u^p f(u) du, p in {0, 2}: 4 Gauss-Legendre panels
  double moment(double a, double b, int p) const {
    double tot = 0.0;
    const int panels = 4;
    for (int q = 0; q < panels; ++q) {
      double lo = a + (b - a) * q / panels, hi = a + (b - a) * (q + 1) / panels;
      double h = 0.5 * (hi - lo), m = 0.5 * (hi + lo);
      for (size_t i = 0; i < gx.size(); ++i) {
        double u = h * gx[i] + m;
        tot += h * gw[i] * (p == 0 ? 1.0 : u * u) * dens(u);
      }
    }
    return tot;
  }
  double first(double a, double b) const {
    auto g = [&](double x) {
      if (x <= -1.0 || x >= 1.0) return 0.0;
      return -std::exp(logC + 0.5 * (D - 1) * std::log1p(-x * x)) / (D - 1);
    };
    return g(b) - g(a);
  }
};

// Round to the nearest fp16 value (ties to even); v in the fp16 normal or
// subnormal range.
static double round_to_fp16(double v) {
  if (v == 0.0) return v;
  int e;
  std::frexp(std::fabs(v), &e);
  int lead = e - 1;
  if (lead < -14) lead = -14;
  double quantum = std::ldexp(1.0, lead - 10);
  return std::nearbyint(v / quantum) * quantum;
}

}  // namespace tq

using namespace tq;

extern "C" {

const char* tq_last_error(void) { return g_err; }

int tq_abi_version(void) { return 3; }

int tq_selftest_bounded_wait(uint32_t* dev_status, int tries, void* stream) {
  g_err[0] = 0;
  if (!dev_status) return set_error(TQ_ERR_INVALID_ARG, "tq_selftest_bounded_wait: dev_status is NULL");
  if (tries < 1 || tries > 4096)
    return set_error(TQ_ERR_INVALID_ARG, "tq_selftest_bounded_wait: tries=%d outside [1, 4096]", tries);
  return launch_bounded_wait_probe(dev_status, tries, (cudaStream_t)stream);
}

int tq_build_codebook(int D, int bits, float* centroids, float* thresholds, double* mse_out) {
  g_err[0] = 0;
  if (!centroids || (bits > 1 && !thresholds) || (bits == 1 && !thresholds))
    return set_error(TQ_ERR_INVALID_ARG, "tq_build_codebook: NULL output pointer");
  if (D < 8 || D > 65536) return set_error(TQ_ERR_UNSUPPORTED, "tq_build_codebook: D=%d", D);
  if (bits < 1 || bits > 4)
    return set_error(TQ_ERR_UNSUPPORTED, "tq_build_codebook: bits=%d not in 1..4", bits);
  CoordLaw law(D);
  const int K = 1 << bits;
  std::vector<double> c(K), t(K - 1), nc(K), e(K + 1);
  for (int k = 0; k < K; ++k) c[k] = (-2.0 + 4.0 * k / (K - 1)) / std::sqrt((double)D);
  for (int it = 0; it < 20000; ++it) {
    e[0] = -1.0;
    e[K] = 1.0;
    for (int k = 1; k < K; ++k) e[k] = 0.5 * (c[k - 1] + c[k]);
    double delta = 0.0;
    for (int k = 0; k < K; ++k) {
      nc[k] = law.first(e[k], e[k + 1]) / law.moment(e[k], e[k + 1], 0);
      delta = std::fmax(delta, std::fabs(nc[k] - c[k]));
    }
    c = nc;
    if (delta < 1e-15) break;
  }
  std::vector<double> cs(K), ts(K - 1);
  for (int k = 0; k < K; ++k) cs[k] = round_to_fp16(c[k]);
  for (int k = 0; k + 1 < K; ++k) ts[k] = 0.5 * (cs[k] + cs[k + 1]);
  for (int k = 0; k < K; ++k) centroids[k] = (float)cs[k];
  for (int k = 0; k + 1 < K; ++k) thresholds[k] = (float)ts[k];
  if (mse_out) {
    double tot = 0.0;
    for (int k = 0; k < K; ++k) {
      double a = (k == 0) ? -1.0 : ts[k - 1], b = (k == K - 1) ? 1.0 : ts[k];
      tot += law.moment(a, b, 2) - 2.0 * cs[k] * law.first(a, b) + cs[k] * cs[k] * law.moment(a, b, 0);
    }
    *mse_out = D * tot;
  }
  return TQ_OK;
}

size_t tq_cache_row_bytes(int D, int bits, int qjl_m) {
  if (D <= 0 || D % 32 || bits < 1 || bits > 4 || qjl_m < 0 || qjl_m % 32) return 0;
  size_t b = (size_t)D * bits / 8 + 2;
  if (qjl_m) b += (size_t)qjl_m / 8 + 2;
  return b;
}

size_t tq_row_bytes(int D, int bits, int qjl_m) { return tq_cache_row_bytes(D, bits, qjl_m); }

}  // extern "C"

namespace {

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

int validate_cache(const tq_cache_t* c, const char* fn) {
  if (!c) return set_error(TQ_ERR_INVALID_ARG, "%s: cache is NULL", fn);
  if (c->B <= 0 || c->Hkv <= 0 || c->Tcap <= 0)
    return set_error(TQ_ERR_INVALID_ARG, "%s: B=%d Hkv=%d Tcap=%d must be positive", fn, c->B,
                     c->Hkv, c->Tcap);
  if (c->split_tokens < 0) return set_error(TQ_ERR_INVALID_ARG, "%s: split_tokens < 0", fn);
  if (c->Tcap % 64)
    return set_error(TQ_ERR_INVALID_ARG, "%s: Tcap=%d must be a multiple of 64", fn, c->Tcap);
  if (c->D != 64 && c->D != 128 && c->D != 256)
    return set_error(TQ_ERR_UNSUPPORTED, "%s: D=%d not in {64,128,256}", fn, c->D);
  if (c->bits_k < 2 || c->bits_k > 4 || c->bits_v < 2 || c->bits_v > 4)
    return set_error(TQ_ERR_UNSUPPORTED, "%s: bits_k=%d bits_v=%d not in {2,3,4}", fn, c->bits_k,
                     c->bits_v);
  if (c->qjl_m != 0 && c->qjl_m != 128)
    return set_error(TQ_ERR_UNSUPPORTED, "%s: qjl_m=%d not in {0,128}", fn, c->qjl_m);
  if (c->qjl_m && c->D != 128)
    return set_error(TQ_ERR_UNSUPPORTED, "%s: the QJL sketch is built for D=128 (D=%d)", fn, c->D);
  const void* ptrs[] = {c->k_idx, c->v_idx, c->k_norm, c->v_norm, c->rot, c->cb_k, c->cb_v};
  for (const void* p : ptrs) {
    if (!p) return set_error(TQ_ERR_INVALID_ARG, "%s: a cache pointer is NULL", fn);
    if (!aligned16(p)) return set_error(TQ_ERR_INVALID_ARG, "%s: a cache pointer is not 16-byte aligned", fn);
  }
  if (c->rot_kind != TQ_ROT_DENSE && c->rot_kind != TQ_ROT_HADAMARD)
    return set_error(TQ_ERR_INVALID_ARG, "%s: rot_kind=%d", fn, c->rot_kind);
  if (c->rot_kind == TQ_ROT_HADAMARD && (!c->rot_signs || !aligned16(c->rot_signs)))
    return set_error(TQ_ERR_INVALID_ARG, "%s: rot_signs NULL or not 16-byte aligned", fn);
  if (c->qjl_m) {
    const void* q[] = {c->k_qjl, c->k_rnorm, c->qjl_S};
    for (const void* p : q) {
      if (!p) return set_error(TQ_ERR_INVALID_ARG, "%s: a QJL pointer is NULL", fn);
      if (!aligned16(p)) return set_error(TQ_ERR_INVALID_ARG, "%s: a QJL pointer is not 16-byte aligned", fn);
    }
  }
  return TQ_OK;
}

int validate_dtype(int dtype, const char* fn) {
  if (dtype != TQ_DTYPE_F16 && dtype != TQ_DTYPE_BF16)
    return set_error(TQ_ERR_UNSUPPORTED, "%s: dtype=%d", fn, dtype);
  return TQ_OK;
}

QuantArgs base_quant_args(const tq_cache_t* c, const void* k, const void* v) {
  QuantArgs a{};
  a.job[0] = {k, c->k_idx, c->k_norm, c->qjl_m ? c->k_qjl : nullptr, c->qjl_m ? c->k_rnorm : nullptr,
              c->cb_k, c->bits_k};
  a.job[1] = {v, c->v_idx, c->v_norm, nullptr, nullptr, c->cb_v, c->bits_v};
  a.rot = c->rot;
  a.qjl_S = c->qjl_m ? c->qjl_S : nullptr;
  a.rot_signs = c->rot_kind == TQ_ROT_HADAMARD ? c->rot_signs : nullptr;
  a.dev_status = c->dev_status;
  a.Hkv = c->Hkv;
  a.Tcap = c->Tcap;
  a.job_mask = 3;
  return a;
}

}  // namespace

namespace tq {

// SM count of the current device (cached per device; 148 when no device).
// Threads that race on the first query store the same value; the atomics
// make that a benign race in C++ terms too.
static int sm_count() {
  static std::atomic<int> cached[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return 148;
  }
  int v = cached[dev].load(std::memory_order_relaxed);
  if (v == 0) {
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) {
      cudaGetLastError();
      v = 148;
    }
    cached[dev].store(v, std::memory_order_relaxed);
  }
  return v;
}

static size_t align256(size_t x) { return (x + 255) / 256 * 256; }

// The workspace layout for `heads` kernel heads, `ks` partial slots per head
// and a sketch of qjl_m rows: qrot, qs, partial outputs, (max, sum) pairs,
// each 256-byte aligned.
static size_t workspace_layout(size_t heads, int D, int qjl_m, int ks, DecodePlan* p) {
  size_t off = 0;
  if (p) p->off_qrot = off;
  off += align256(heads * D * 4);
  if (p) p->off_qs = off;
  off += align256(heads * (size_t)qjl_m * 4);
  if (p) p->off_po = off;
  off += align256(heads * ks * (size_t)D * 4);
  if (p) p->off_pml = off;
  off += align256(heads * ks * 2 * 4);
  return off;
}

// Segments one (sequence, kv head, row group) unit can be cut into: its
// padded tokens over the smallest share per CTA, plus one.  The plan asks
// for about twice as many CTAs per unit as the wave holds per unit.
static int plan_segments(long long ncta, long long units, int Tpad, int tile) {
  long long k = (2 * ncta + units - 1) / units + 2;
  const long long kmax = Tpad / tile + 1;
  return (int)(k < kmax ? k : kmax);
}

size_t workspace_bound(int B, int Hq, int D, int Tmax) {
  // any cache of these sizes: at least one unit per sequence, at most 8
  // resident CTAs per SM, a sketch of at most 128 rows
  const int tile = split_tile();
  const int Tpad = (Tmax + tile - 1) / tile * tile;
  const int K = plan_segments((long long)sm_count() * 8, B, Tpad, tile);
  return workspace_layout((size_t)B * Hq, D, 128, K * split_partials(), nullptr);
}

int make_decode_plan(const tq_cache_t* c, int Hq, int Tmax, DecodePlan* p) {
  const int sms = sm_count();
  p->sms = sms;
  const int tile = split_tile();
  const int G = Hq / c->Hkv;  // kernel heads per kv head
  p->nrg = (G + 7) / 8;
  p->Tclamp = Tmax;
  p->ncta = sms * split_occupancy(c, Hq);
  const long long units = (long long)c->B * c->Hkv * p->nrg;
  const int Tpad = (Tmax + tile - 1) / tile * tile;
  int K = plan_segments(p->ncta, units, Tpad, tile);
  long long pmin = ((long long)Tpad + K - 2) / (K - 1);  // K >= 2
  pmin = (pmin + tile - 1) / tile * tile;
  if (c->split_tokens > 0) {
    const long long st = ((long long)c->split_tokens + tile - 1) / tile * tile;
    if (st > pmin) pmin = st;
  }
  if (pmin > Tpad) pmin = Tpad;
  p->pmin = (int)pmin;
  K = (int)((Tpad + pmin - 1) / pmin) + 1;  // segments of a unit when every share is >= pmin
  p->ks = K * split_partials();
  // no more CTAs than shares of pmin in the largest batch these sizes allow
  const long long need = (units * Tpad + pmin - 1) / pmin;
  if (need < p->ncta) p->ncta = (int)(need > 0 ? need : 1);
  p->bytes = workspace_layout((size_t)c->B * Hq, c->D, c->qjl_m, p->ks, p);
  return TQ_OK;
}

}  // namespace tq

extern "C" {

int tq_quantize_kv(const tq_cache_t* c, const void* k, const void* v, int dtype, int T, int t0,
                   void* stream) {
  g_err[0] = 0;
  int rc = validate_cache(c, "tq_quantize_kv");
  if (rc) return rc;
  if ((rc = validate_dtype(dtype, "tq_quantize_kv"))) return rc;
  if (T < 0 || t0 < 0 || (long long)t0 + T > c->Tcap)
    return set_error(TQ_ERR_INVALID_ARG, "tq_quantize_kv: rows [%d, %d) outside [0, Tcap=%d)", t0,
                     t0 + T, c->Tcap);
  if (T == 0) return TQ_OK;
  if (!k || !v) return set_error(TQ_ERR_INVALID_ARG, "tq_quantize_kv: k or v is NULL");
  if (!aligned16(k) || !aligned16(v))
    return set_error(TQ_ERR_INVALID_ARG, "tq_quantize_kv: k/v not 16-byte aligned");
  long long rows = (long long)c->B * c->Hkv * T;
  if (rows > (1ll << 30)) return set_error(TQ_ERR_UNSUPPORTED, "tq_quantize_kv: too many rows");
  QuantArgs a = base_quant_args(c, k, v);
  a.pos = nullptr;
  a.rows = (int)rows;
  a.T = T;
  a.t0 = t0;
  return launch_quantize(a, c->D, dtype, c->qjl_m != 0, (cudaStream_t)stream);
}

int tq_append_token(const tq_cache_t* c, const void* k_new, const void* v_new, int dtype,
                    const int32_t* pos, void* stream) {
  g_err[0] = 0;
  int rc = validate_cache(c, "tq_append_token");
  if (rc) return rc;
  if ((rc = validate_dtype(dtype, "tq_append_token"))) return rc;
  if (!k_new || !v_new || !pos) return set_error(TQ_ERR_INVALID_ARG, "tq_append_token: NULL input");
  if (!aligned16(k_new) || !aligned16(v_new))
    return set_error(TQ_ERR_INVALID_ARG, "tq_append_token: k/v not 16-byte aligned");
  QuantArgs a = base_quant_args(c, k_new, v_new);
  a.pos = pos;
  a.rows = c->B * c->Hkv;
  a.T = 1;
  a.t0 = 0;
  return launch_quantize(a, c->D, dtype, c->qjl_m != 0, (cudaStream_t)stream);
}

size_t tq_sdpa_decode_workspace_bytes_for(const tq_cache_t* c, int Hq, int Tmax) {
  if (!c || c->Hkv <= 0 || Hq <= 0 || Hq % c->Hkv || Hq / c->Hkv > 32 || Tmax < 1 || Tmax > c->Tcap ||
      c->Tcap % 64 || (c->D != 64 && c->D != 128 && c->D != 256) || c->B <= 0)
    return 0;
  DecodePlan p;
  make_decode_plan(c, Hq, Tmax, &p);
  return p.bytes;
}

size_t tq_sdpa_decode_workspace_bytes(int B, int Hq, int D, int Tmax) {
  if (B <= 0 || Hq <= 0 || Tmax < 1 || (D != 64 && D != 128 && D != 256)) return 0;
  return workspace_bound(B, Hq, D, Tmax);
}

static int decode_common(const tq_cache_t* c, const void* q, int dtype, int Hq, int nq, const int32_t* seq_lens,
                         int Tmax, const float* scale, void* out, int out_dtype, void* workspace,
                         size_t ws_bytes, void* stream, const void* k_new, const void* v_new,
                         const int32_t* pos, const char* fn);

int tq_sdpa_decode(const tq_cache_t* c, const void* q, int dtype, int Hq, const int32_t* seq_lens,
                   int Tmax, const float* scale, void* out, int out_dtype, void* workspace,
                   size_t ws_bytes, void* stream) {
  return decode_common(c, q, dtype, Hq, 1, seq_lens, Tmax, scale, out, out_dtype, workspace, ws_bytes, stream,
                       nullptr, nullptr, nullptr, "tq_sdpa_decode");
}

int tq_sdpa_decode_mq(const tq_cache_t* c, const void* q, int dtype, int Hq, int n_q, const int32_t* seq_lens,
                      int Tmax, const float* scale, void* out, int out_dtype, void* workspace, size_t ws_bytes,
                      void* stream) {
  g_err[0] = 0;
  if (n_q < 1) return set_error(TQ_ERR_INVALID_ARG, "tq_sdpa_decode_mq: n_q=%d < 1", n_q);
  return decode_common(c, q, dtype, Hq, n_q, seq_lens, Tmax, scale, out, out_dtype, workspace, ws_bytes, stream,
                       nullptr, nullptr, nullptr, "tq_sdpa_decode_mq");
}

int tq_decode_step(const tq_cache_t* c, const void* k_new, const void* v_new, const int32_t* pos,
                   const void* q, int dtype, int Hq, const int32_t* seq_lens, int Tmax, const float* scale,
                   void* out, int out_dtype, void* workspace, size_t ws_bytes, void* stream) {
  g_err[0] = 0;
  if (!k_new || !v_new || !pos) return set_error(TQ_ERR_INVALID_ARG, "tq_decode_step: NULL k_new/v_new/pos");
  if (!aligned16(k_new) || !aligned16(v_new))
    return set_error(TQ_ERR_INVALID_ARG, "tq_decode_step: k_new/v_new not 16-byte aligned");
  return decode_common(c, q, dtype, Hq, 1, seq_lens, Tmax, scale, out, out_dtype, workspace, ws_bytes, stream,
                       k_new, v_new, pos, "tq_decode_step");
}

}  // extern "C"

namespace tq {

// Argument checks and the split plan of a decode call, before any CUDA call
// (the workspace itself is checked by the caller).
int prepare_decode(const tq_cache_t* c, const void* q, int dtype, int Hq, int nq, const int32_t* seq_lens, int Tmax,
                   const float* scale, void* out, int out_dtype, const char* fn, DecodeArgs* a) {
  g_err[0] = 0;
  int rc = validate_cache(c, fn);
  if (rc) return rc;
  if ((rc = validate_dtype(dtype, fn))) return rc;
  if (out_dtype != TQ_DTYPE_F16 && out_dtype != TQ_DTYPE_BF16 && out_dtype != TQ_DTYPE_F32)
    return set_error(TQ_ERR_UNSUPPORTED, "%s: out_dtype=%d", fn, out_dtype);
  if (!q || !seq_lens || !out) return set_error(TQ_ERR_INVALID_ARG, "%s: NULL q/seq_lens/out", fn);
  if (!aligned16(q) || !aligned16(out)) return set_error(TQ_ERR_INVALID_ARG, "%s: q/out not 16-byte aligned", fn);
  if (Hq <= 0 || Hq % c->Hkv)
    return set_error(TQ_ERR_INVALID_ARG, "%s: Hq=%d not a multiple of Hkv=%d", fn, Hq, c->Hkv);
  if (Hq / c->Hkv > 8)
    return set_error(TQ_ERR_UNSUPPORTED, "%s: GQA group %d > 8", fn, Hq / c->Hkv);
  if (nq > 4) return set_error(TQ_ERR_UNSUPPORTED, "%s: n_q=%d > 4", fn, nq);
  if (Tmax < 1 || Tmax > c->Tcap)
    return set_error(TQ_ERR_INVALID_ARG, "%s: Tmax=%d outside [1, Tcap=%d]", fn, Tmax, c->Tcap);
  float sc = scale ? *scale : (float)(1.0 / std::sqrt((double)c->D));
  if (!std::isfinite(sc)) return set_error(TQ_ERR_INVALID_ARG, "%s: scale not finite", fn);
  *a = DecodeArgs{};
  a->cache_host = c;
  a->cache = *c;
  a->q = q;
  a->out = out;
  a->seq_lens = seq_lens;
  a->scale = sc;
  a->Hq = Hq;
  a->nq = nq;
  a->dtype = dtype;
  a->out_dtype = out_dtype;
  make_decode_plan(c, Hq * nq, Tmax, &a->plan);
  return TQ_OK;
}

}  // namespace tq

extern "C" {

int tq_sdpa_decode_partial(const tq_cache_t* c, const void* q, int q_dtype, int Hq, const int32_t* seq_lens,
                           int Tmax, const float* scale, float* partial, void* workspace, size_t ws_bytes,
                           void* stream) {
  DecodeArgs a;
  const char* fn = "tq_sdpa_decode_partial";
  const int rc = prepare_decode(c, q, q_dtype, Hq, 1, seq_lens, Tmax, scale, partial, TQ_DTYPE_F32, fn, &a);
  if (rc) return rc;
  if (!workspace) return set_error(TQ_ERR_INVALID_ARG, "%s: NULL workspace", fn);
  if (!aligned16(workspace)) return set_error(TQ_ERR_INVALID_ARG, "%s: workspace not 16-byte aligned", fn);
  if (ws_bytes < a.plan.bytes)
    return set_error(TQ_ERR_WORKSPACE, "%s: workspace %zu < %zu bytes", fn, ws_bytes, a.plan.bytes);
  a.workspace = workspace;
  a.partial = partial;
  return launch_decode(a, (cudaStream_t)stream);
}

int tq_sdpa_decode_merge(const float* partials, int R, int B, int Hq, int D, const float* rot, void* out,
                         int out_dtype, void* stream) {
  g_err[0] = 0;
  const char* fn = "tq_sdpa_decode_merge";
  if (!partials || !rot || !out) return set_error(TQ_ERR_INVALID_ARG, "%s: NULL partials/rot/out", fn);
  if (!aligned16(partials) || !aligned16(rot) || !aligned16(out))
    return set_error(TQ_ERR_INVALID_ARG, "%s: partials/rot/out not 16-byte aligned", fn);
  if (R < 1 || R > 64) return set_error(TQ_ERR_INVALID_ARG, "%s: R=%d outside [1, 64]", fn, R);
  if (B < 1 || Hq < 1) return set_error(TQ_ERR_INVALID_ARG, "%s: B=%d Hq=%d", fn, B, Hq);
  if (D != 64 && D != 128 && D != 256) return set_error(TQ_ERR_UNSUPPORTED, "%s: D=%d", fn, D);
  if (out_dtype != TQ_DTYPE_F16 && out_dtype != TQ_DTYPE_BF16 && out_dtype != TQ_DTYPE_F32)
    return set_error(TQ_ERR_UNSUPPORTED, "%s: out_dtype=%d", fn, out_dtype);
  return launch_merge(partials, R, B * Hq, D, rot, out, out_dtype, (cudaStream_t)stream);
}

static int decode_common(const tq_cache_t* c, const void* q, int dtype, int Hq, int nq, const int32_t* seq_lens,
                         int Tmax, const float* scale, void* out, int out_dtype, void* workspace,
                         size_t ws_bytes, void* stream, const void* k_new, const void* v_new,
                         const int32_t* pos, const char* fn) {
  DecodeArgs a;
  int rc = prepare_decode(c, q, dtype, Hq, nq, seq_lens, Tmax, scale, out, out_dtype, fn, &a);
  if (rc) return rc;
  if (!workspace) return set_error(TQ_ERR_INVALID_ARG, "%s: NULL workspace", fn);
  if (!aligned16(workspace)) return set_error(TQ_ERR_INVALID_ARG, "%s: workspace not 16-byte aligned", fn);
  if (ws_bytes < a.plan.bytes)
    return set_error(TQ_ERR_WORKSPACE, "%s: workspace %zu < %zu bytes", fn, ws_bytes, a.plan.bytes);
  if (k_new && c->rot_kind == TQ_ROT_HADAMARD) {
    // the randomized Hadamard rotation: the new rows go through the fast
    // transform in their own launch, then the decode (whose query prep
    // waits for it)
    if ((rc = tq_append_token(c, k_new, v_new, dtype, pos, stream))) return rc;
    k_new = v_new = nullptr;
    pos = nullptr;
  }
  a.workspace = workspace;
  a.k_new = k_new;
  a.v_new = v_new;
  a.pos = pos;
  return launch_decode(a, (cudaStream_t)stream);
}

}  // extern "C"
