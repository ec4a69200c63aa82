// nq_abi.cu -- the extern "C" boundary of libnq: argument validation, RoPE
// table construction on the host, status codes and error messages.  Every
// compute entry point validates all sizes, strides and alignments on the host
// and launches nothing when they are wrong.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <string>

#include "nq_internal.h"

namespace {

thread_local std::string g_last_error = "no error";

nq_status fail(nq_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

nq_status cuda_status(cudaError_t err, const char* what) {
  if (err == cudaSuccess) return NQ_OK;
  return fail(NQ_ERR_CUDA, "%s: %s", what, cudaGetErrorString(err));
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

nq_status check_kv(const void* p, nq_kv_strides s, const char* name) {
  if (!p) return fail(NQ_ERR_INVALID, "%s is NULL", name);
  if (!aligned(p, 16)) return fail(NQ_ERR_INVALID, "%s must be 16-byte aligned", name);
  if (s.unit < 0 || s.head < 0 || s.token < 0 || s.unit % 8 || s.head % 8 || s.token % 8)
    return fail(NQ_ERR_INVALID, "%s strides must be non-negative multiples of 8 elements", name);
  return NQ_OK;
}

nq_status check_packed(const nq_packed* p, const char* name) {
  if (!p) return fail(NQ_ERR_INVALID, "%s descriptor is NULL", name);
  if (p->bits != 2 && p->bits != 3)
    return fail(NQ_ERR_INVALID, "%s.bits must be 2 or 3 (got %d)", name, p->bits);
  if (!p->codes || !p->meta) return fail(NQ_ERR_INVALID, "%s codes/meta is NULL", name);
  if (!aligned(p->codes, 16)) return fail(NQ_ERR_INVALID, "%s.codes must be 16-byte aligned", name);
  if (!aligned(p->meta, 4)) return fail(NQ_ERR_INVALID, "%s.meta must be 4-byte aligned", name);
  if (p->unit_stride < 0 || p->head_stride < 0)
    return fail(NQ_ERR_INVALID, "%s strides must be non-negative", name);
  return NQ_OK;
}

nq_status check_rope(const float* tab, int64_t max_pos) {
  if (!tab) return fail(NQ_ERR_INVALID, "rope_tab is NULL (required for keys)");
  if (!aligned(tab, 16)) return fail(NQ_ERR_INVALID, "rope_tab must be 16-byte aligned");
  if (max_pos < 1) return fail(NQ_ERR_INVALID, "rope_max_pos must be >= 1");
  return NQ_OK;
}

constexpr int64_t kMaxSelectT = int64_t(1) << 20;

// The address at which the device reads p: p itself for device (or managed)
// memory, the mapped address for pinned host memory; anything the device
// cannot read (plain host memory) is refused before any launch.
nq_status device_readable(const void* p, const void** out, const char* name) {
  cudaPointerAttributes attr{};
  if (cudaPointerGetAttributes(&attr, p) != cudaSuccess) {
    cudaGetLastError();  // clear the sticky-free error of the query
    return fail(NQ_ERR_INVALID, "%s: the device cannot read this pointer", name);
  }
  if (attr.type == cudaMemoryTypeDevice || attr.type == cudaMemoryTypeManaged) {
    *out = p;
    return NQ_OK;
  }
  if (attr.type == cudaMemoryTypeHost && attr.devicePointer) {
    *out = attr.devicePointer;
    return NQ_OK;
  }
  return fail(NQ_ERR_INVALID, "%s is host memory the device cannot read (not pinned/mapped)", name);
}

}  // namespace

extern "C" {

const char* nq_last_error(void) { return g_last_error.c_str(); }

int nq_version(void) { return 1; }

int64_t nq_packed_bytes_per_vector(int bits) {
  if (bits != 2 && bits != 3) return -1;
  return 4 * (4 * bits) + 4;
}

size_t nq_rope_tables_bytes(int64_t max_pos) {
  if (max_pos < 1) return 0;
  const int64_t na = (max_pos + 255) / 256;
  return static_cast<size_t>(na + 256) * nq::kHalf * 2 * sizeof(float);
}

nq_status nq_rope_tables_fill_host(double theta, int64_t max_pos, void* host_buf, size_t bytes) {
  if (!(theta > 1.0) || !std::isfinite(theta)) return fail(NQ_ERR_INVALID, "theta must be > 1");
  if (max_pos < 1) return fail(NQ_ERR_INVALID, "max_pos must be >= 1");
  if (!host_buf) return fail(NQ_ERR_INVALID, "host_buf is NULL");
  if (bytes < nq_rope_tables_bytes(max_pos))
    return fail(NQ_ERR_WORKSPACE, "rope table buffer too small: %zu < %zu", bytes,
                nq_rope_tables_bytes(max_pos));
  float* t = static_cast<float*>(host_buf);
  const int64_t na = (max_pos + 255) / 256;
  for (int i = 0; i < nq::kHalf; ++i) {
    // w_i = theta^(-2i/D) with D = 128
    const double w = std::pow(theta, -static_cast<double>(i) / 64.0);
    for (int64_t a = 0; a < na; ++a) {
      const double ang = static_cast<double>(256 * a) * w;
      t[2 * (a * nq::kHalf + i)] = static_cast<float>(std::cos(ang));
      t[2 * (a * nq::kHalf + i) + 1] = static_cast<float>(std::sin(ang));
    }
    for (int64_t b = 0; b < 256; ++b) {
      const double ang = static_cast<double>(b) * w;
      t[2 * ((na + b) * nq::kHalf + i)] = static_cast<float>(std::cos(ang));
      t[2 * ((na + b) * nq::kHalf + i) + 1] = static_cast<float>(std::sin(ang));
    }
  }
  return NQ_OK;
}

size_t nq_score_workspace_bytes(int units, int heads) {
  if (units < 0 || heads < 0) return 0;
  return static_cast<size_t>(units) * heads * nq::kD * sizeof(float);
}

nq_status nq_score(const void* K, nq_kv_strides ks, int units, int heads, int64_t T, int W,
                   double* scores, void* ws, size_t ws_bytes, nq_stream_t stream) {
  if (units < 0 || heads < 1 || heads > 1024)
    return fail(NQ_ERR_INVALID, "need units >= 0 and 1 <= heads <= 1024");
  if (T < 1 || W < 1 || W > T) return fail(NQ_ERR_INVALID, "need 1 <= W <= T");
  if (heads > 128) return fail(NQ_ERR_UNSUPPORTED, "nq_score supports at most 128 heads");
  if (units == 0) return NQ_OK;
  if (nq_status st = check_kv(K, ks, "K")) return st;
  if (!scores || !aligned(scores, 8)) return fail(NQ_ERR_INVALID, "scores NULL or misaligned");
  if (!ws || !aligned(ws, 16)) return fail(NQ_ERR_INVALID, "workspace NULL or not 16-byte aligned");
  if (ws_bytes < nq_score_workspace_bytes(units, heads))
    return fail(NQ_ERR_WORKSPACE, "score workspace too small: %zu < %zu", ws_bytes,
                nq_score_workspace_bytes(units, heads));
  if (static_cast<int64_t>(units) * ((T + 127) / 128) > 0x7FFFFFFF)
    return fail(NQ_ERR_UNSUPPORTED, "units * T too large for one launch");
  if (static_cast<int64_t>(units) * heads > 0x7FFFFFFF)
    return fail(NQ_ERR_UNSUPPORTED, "units * heads too large for one launch");
  return cuda_status(nq::launch_score(K, ks, units, heads, T, W, scores, static_cast<float*>(ws),
                                      reinterpret_cast<cudaStream_t>(stream)),
                     "nq_score launch");
}

nq_status nq_score_static(const void* K, nq_kv_strides ks, int units, int heads, int64_t T, int W,
                          double* scores, nq_stream_t stream) {
  if (units < 0 || heads < 1 || heads > 1024)
    return fail(NQ_ERR_INVALID, "need units >= 0 and 1 <= heads <= 1024");
  if (T < 1 || W < 1 || W > T) return fail(NQ_ERR_INVALID, "need 1 <= W <= T");
  if (heads > 128) return fail(NQ_ERR_UNSUPPORTED, "nq_score_static supports at most 128 heads");
  if (static_cast<int64_t>(units) * heads > NQ_SCORE_STATIC_MAX_VECTORS)
    return fail(NQ_ERR_UNSUPPORTED,
                "nq_score_static: units * heads = %lld exceeds its fixed scratch of %d "
                "(unit, head) window means; use nq_score with a caller workspace",
                static_cast<long long>(units) * heads, NQ_SCORE_STATIC_MAX_VECTORS);
  if (units == 0) return NQ_OK;
  if (nq_status st = check_kv(K, ks, "K")) return st;
  if (!scores || !aligned(scores, 8)) return fail(NQ_ERR_INVALID, "scores NULL or misaligned");
  if (static_cast<int64_t>(units) * ((T + 127) / 128) > 0x7FFFFFFF)
    return fail(NQ_ERR_UNSUPPORTED, "units * T too large for one launch");
  return cuda_status(nq::launch_score_static(K, ks, units, heads, T, W, scores,
                                             reinterpret_cast<cudaStream_t>(stream)),
                     "nq_score_static");
}

int64_t nq_kept_count(int64_t T, int64_t W, int evict_pct) {
  if (T < 0 || W < 0) return -1;
  if (T <= 1 + W || evict_pct <= 0) return T;
  const int64_t mid = T - 1 - W;
  const int pct = evict_pct > 100 ? 100 : evict_pct;
  return T - (mid * pct) / 100;
}

nq_status nq_select(const double* scores, int units, int64_t T, int W, int evict_pct,
                    int32_t* kept, int64_t kept_stride, nq_stream_t stream) {
  if (units < 0 || T < 1 || W < 0 || W > T)
    return fail(NQ_ERR_INVALID, "need units >= 0, T >= 1, 0 <= W <= T");
  if (evict_pct < 0 || evict_pct > 100) return fail(NQ_ERR_INVALID, "evict_pct must be in [0, 100]");
  if (T > kMaxSelectT)
    return fail(NQ_ERR_UNSUPPORTED, "T = %lld exceeds the selection limit %lld",
                static_cast<long long>(T), static_cast<long long>(kMaxSelectT));
  if (units == 0) return NQ_OK;
  if (!scores || !aligned(scores, 8)) return fail(NQ_ERR_INVALID, "scores NULL or misaligned");
  if (!kept || !aligned(kept, 4)) return fail(NQ_ERR_INVALID, "kept NULL or misaligned");
  const int64_t n = nq_kept_count(T, W, evict_pct);
  if (kept_stride < n)
    return fail(NQ_ERR_INVALID, "kept_stride %lld < kept count %lld",
                static_cast<long long>(kept_stride), static_cast<long long>(n));
  return cuda_status(nq::launch_select(scores, units, T, W, evict_pct, n, kept, kept_stride,
                                       reinterpret_cast<cudaStream_t>(stream)),
                     "nq_select launch");
}

// The exact layout travels as an nq_packed whose meta points to the uint16
// scales (checked here for 2-byte alignment).
static nq_packed from_exact(const nq_packed_exact* p) {
  nq_packed q{};
  if (p) {
    q.codes = p->codes;
    q.meta = reinterpret_cast<uint32_t*>(p->sigma);
    q.unit_stride = p->unit_stride;
    q.head_stride = p->head_stride;
    q.bits = p->bits;
  }
  return q;
}

static nq_status check_store(const nq_packed* p, bool exact, const char* name) {
  if (!p) return fail(NQ_ERR_INVALID, "%s descriptor is NULL", name);
  if (!exact) return check_packed(p, name);
  if (p->bits != 2 && p->bits != 3)
    return fail(NQ_ERR_INVALID, "%s.bits must be 2 or 3 (got %d)", name, p->bits);
  if (!p->codes || !p->meta) return fail(NQ_ERR_INVALID, "%s codes/sigma is NULL", name);
  if (!aligned(p->codes, 16)) return fail(NQ_ERR_INVALID, "%s.codes must be 16-byte aligned", name);
  if (!aligned(p->meta, 2)) return fail(NQ_ERR_INVALID, "%s.sigma must be 2-byte aligned", name);
  if (p->unit_stride < 0 || p->head_stride < 0)
    return fail(NQ_ERR_INVALID, "%s strides must be non-negative", name);
  return NQ_OK;
}

static nq_status encode_impl(const void* K, nq_kv_strides ks, const void* V, nq_kv_strides vs, int units,
                      int heads, int64_t T_in, int64_t n, const int32_t* kept,
                      int64_t kept_stride, int64_t pos_base, const float* rope_tab,
                      int64_t rope_max_pos, const nq_packed* k_out, const nq_packed* v_out,
                      int64_t slot0, bool exact, nq_stream_t stream) {
  if (!K && !V) return fail(NQ_ERR_INVALID, "K and V are both NULL");
  if (units < 0 || heads < 1 || heads > 1024 || n < 0 || slot0 < 0 || pos_base < 0)
    return fail(NQ_ERR_INVALID, "need units >= 0, 1 <= heads <= 1024, n >= 0, slot0 >= 0, pos_base >= 0");
  if (units == 0 || n == 0) return NQ_OK;
  if (T_in < 1) return fail(NQ_ERR_INVALID, "T_in must be >= 1");
  if (static_cast<int64_t>(units) * n >= (int64_t(1) << 31))
    return fail(NQ_ERR_UNSUPPORTED, "units * n must stay below 2^31 (slot pairs of one call)");
  if (kept) {
    if (!aligned(kept, 4)) return fail(NQ_ERR_INVALID, "kept misaligned");
    if (kept_stride < n) return fail(NQ_ERR_INVALID, "kept_stride < n");
  } else if (n > T_in) {
    return fail(NQ_ERR_INVALID, "n > T_in without a kept list");
  }
  if (K) {
    if (nq_status st = check_kv(K, ks, "K")) return st;
    if (nq_status st = check_store(k_out, exact, "k_out")) return st;
    if (nq_status st = check_rope(rope_tab, rope_max_pos)) return st;
    if (!kept && pos_base + n > rope_max_pos)
      return fail(NQ_ERR_INVALID, "positions up to %lld exceed rope_max_pos %lld",
                  static_cast<long long>(pos_base + n - 1), static_cast<long long>(rope_max_pos));
  }
  if (V) {
    if (nq_status st = check_kv(V, vs, "V")) return st;
    if (nq_status st = check_store(v_out, exact, "v_out")) return st;
  }
  // K and V may live in pinned host memory: the kernels then read only the
  // rows they encode across the bus
  const void* Kd = nullptr;
  const void* Vd = nullptr;
  if (K)
    if (nq_status st = device_readable(K, &Kd, "K")) return st;
  if (V)
    if (nq_status st = device_readable(V, &Vd, "V")) return st;
  nq::EncodeLaunch L{};
  L.K = Kd;
  L.ks = ks;
  L.V = Vd;
  L.vs = vs;
  L.units = units;
  L.heads = heads;
  L.T_in = T_in;
  L.n = n;
  L.kept = kept;
  L.kept_stride = kept_stride;
  L.pos_base = pos_base;
  L.rope_tab = rope_tab;
  L.rope_max_pos = rope_max_pos;
  if (K) L.k_out = *k_out;
  if (V) L.v_out = *v_out;
  L.slot0 = slot0;
  L.exact = exact;
  return cuda_status(nq::launch_encode(L, reinterpret_cast<cudaStream_t>(stream)),
                     exact ? "nq_encode_exact launch" : "nq_encode launch");
}

nq_status nq_encode(const void* K, nq_kv_strides ks, const void* V, nq_kv_strides vs, int units,
                    int heads, int64_t T_in, int64_t n, const int32_t* kept, int64_t kept_stride,
                    int64_t pos_base, const float* rope_tab, int64_t rope_max_pos,
                    const nq_packed* k_out, const nq_packed* v_out, int64_t slot0,
                    nq_stream_t stream) {
  return encode_impl(K, ks, V, vs, units, heads, T_in, n, kept, kept_stride, pos_base, rope_tab,
                     rope_max_pos, k_out, v_out, slot0, false, stream);
}

nq_status nq_encode_exact(const void* K, nq_kv_strides ks, const void* V, nq_kv_strides vs,
                          int units, int heads, int64_t T_in, int64_t n, const int32_t* kept,
                          int64_t kept_stride, int64_t pos_base, const float* rope_tab,
                          int64_t rope_max_pos, const nq_packed_exact* k_out,
                          const nq_packed_exact* v_out, int64_t slot0, nq_stream_t stream) {
  const nq_packed k = from_exact(k_out), v = from_exact(v_out);
  return encode_impl(K, ks, V, vs, units, heads, T_in, n, kept, kept_stride, pos_base, rope_tab,
                     rope_max_pos, k_out ? &k : nullptr, v_out ? &v : nullptr, slot0, true,
                     stream);
}

static nq_status decode_impl(const nq_packed* k_in, const nq_packed* v_in, int units, int heads,
                             int64_t n, int64_t slot0, const int32_t* positions,
                             int64_t pos_stride, int64_t pos_base, const float* rope_tab,
                             int64_t rope_max_pos, void* K_out, nq_kv_strides kos, void* V_out,
                             nq_kv_strides vos, bool exact, nq_stream_t stream) {
  if (!K_out && !V_out) return fail(NQ_ERR_INVALID, "K_out and V_out are both NULL");
  if (units < 0 || heads < 1 || heads > 1024 || n < 0 || slot0 < 0 || pos_base < 0)
    return fail(NQ_ERR_INVALID, "need units >= 0, 1 <= heads <= 1024, n >= 0, slot0 >= 0, pos_base >= 0");
  if (units == 0 || n == 0) return NQ_OK;
  if (positions) {
    if (!aligned(positions, 4)) return fail(NQ_ERR_INVALID, "positions misaligned");
    if (pos_stride < n) return fail(NQ_ERR_INVALID, "pos_stride < n");
  }
  if (K_out) {
    if (nq_status st = check_kv(K_out, kos, "K_out")) return st;
    if (nq_status st = check_store(k_in, exact, "k_in")) return st;
    if (nq_status st = check_rope(rope_tab, rope_max_pos)) return st;
    if (!positions && pos_base + n > rope_max_pos)
      return fail(NQ_ERR_INVALID, "positions up to %lld exceed rope_max_pos %lld",
                  static_cast<long long>(pos_base + n - 1), static_cast<long long>(rope_max_pos));
  }
  if (V_out) {
    if (nq_status st = check_kv(V_out, vos, "V_out")) return st;
    if (nq_status st = check_store(v_in, exact, "v_in")) return st;
  }
  nq::DecodeLaunch L{};
  L.exact = exact;
  if (K_out) L.k_in = *k_in;
  if (V_out) L.v_in = *v_in;
  L.units = units;
  L.heads = heads;
  L.n = n;
  L.slot0 = slot0;
  L.positions = positions;
  L.pos_stride = pos_stride;
  L.pos_base = pos_base;
  L.rope_tab = rope_tab;
  L.rope_max_pos = rope_max_pos;
  L.K_out = K_out;
  L.kos = kos;
  L.V_out = V_out;
  L.vos = vos;
  return cuda_status(nq::launch_decode(L, reinterpret_cast<cudaStream_t>(stream)),
                     exact ? "nq_decode_exact launch" : "nq_decode launch");
}

nq_status nq_decode(const nq_packed* k_in, const nq_packed* v_in, int units, int heads,
                    int64_t n, int64_t slot0, const int32_t* positions, int64_t pos_stride,
                    int64_t pos_base, const float* rope_tab, int64_t rope_max_pos, void* K_out,
                    nq_kv_strides kos, void* V_out, nq_kv_strides vos, nq_stream_t stream) {
  return decode_impl(k_in, v_in, units, heads, n, slot0, positions, pos_stride, pos_base,
                     rope_tab, rope_max_pos, K_out, kos, V_out, vos, false, stream);
}

nq_status nq_decode_exact(const nq_packed_exact* k_in, const nq_packed_exact* v_in, int units,
                          int heads, int64_t n, int64_t slot0, const int32_t* positions,
                          int64_t pos_stride, int64_t pos_base, const float* rope_tab,
                          int64_t rope_max_pos, void* K_out, nq_kv_strides kos, void* V_out,
                          nq_kv_strides vos, nq_stream_t stream) {
  const nq_packed k = from_exact(k_in), v = from_exact(v_in);
  return decode_impl(k_in ? &k : nullptr, v_in ? &v : nullptr, units, heads, n, slot0, positions,
                     pos_stride, pos_base, rope_tab, rope_max_pos, K_out, kos, V_out, vos, true,
                     stream);
}

int64_t nq_packed_exact_bytes_per_vector(int bits) {
  if (bits != 2 && bits != 3) return -1;
  return 4 * (4 * bits) + 2;
}

size_t nq_attend_workspace_bytes(int units, int heads, int G, int64_t n) {
  if (units < 0 || heads < 1 || G < 1 || n < 1) return 0;
  return nq::attend_workspace_floats(units, heads, G, n) * sizeof(float);
}

nq_status nq_attend(const float* q, int units, int heads, int G, const nq_packed* k_in,
                    const nq_packed* v_in, int64_t n, int64_t slot0, const int32_t* positions,
                    int64_t pos_stride, int64_t pos_base, const float* rope_tab,
                    int64_t rope_max_pos, float scale, float* out, float* lse, void* ws,
                    size_t ws_bytes, nq_stream_t stream) {
  if (units < 0 || heads < 1 || heads > 1024 || G < 1 || G > 8)
    return fail(NQ_ERR_INVALID, "need units >= 0, 1 <= heads <= 1024, 1 <= G <= 8");
  if (n < 1 || slot0 < 0 || pos_base < 0)
    return fail(NQ_ERR_INVALID, "need n >= 1, slot0 >= 0, pos_base >= 0");
  if (!std::isfinite(scale)) return fail(NQ_ERR_INVALID, "scale must be finite");
  if (units == 0) return NQ_OK;
  if (!q || !aligned(q, 16)) return fail(NQ_ERR_INVALID, "q NULL or not 16-byte aligned");
  if (!out || !aligned(out, 4)) return fail(NQ_ERR_INVALID, "out NULL or misaligned");
  if (lse && !aligned(lse, 4)) return fail(NQ_ERR_INVALID, "lse misaligned");
  if (nq_status st = check_packed(k_in, "k_in")) return st;
  if (nq_status st = check_packed(v_in, "v_in")) return st;
  if (nq_status st = check_rope(rope_tab, rope_max_pos)) return st;
  if (positions) {
    if (!aligned(positions, 4)) return fail(NQ_ERR_INVALID, "positions misaligned");
    if (pos_stride < n) return fail(NQ_ERR_INVALID, "pos_stride < n");
  } else if (pos_base + n > rope_max_pos) {
    return fail(NQ_ERR_INVALID, "positions up to %lld exceed rope_max_pos %lld",
                static_cast<long long>(pos_base + n - 1), static_cast<long long>(rope_max_pos));
  }
  if (!ws || !aligned(ws, 16)) return fail(NQ_ERR_INVALID, "workspace NULL or not 16-byte aligned");
  const size_t need = nq_attend_workspace_bytes(units, heads, G, n);
  if (ws_bytes < need)
    return fail(NQ_ERR_WORKSPACE, "attend workspace too small: %zu < %zu", ws_bytes, need);
  if (n > 0x7FFFFFFF || nq::attend_ctas(units, heads, n) > 0x7FFFFFFF ||
      static_cast<int64_t>(units) * heads * G > 0x7FFFFFFF)
    return fail(NQ_ERR_UNSUPPORTED, "n or units * heads * chunks too large for one launch");
  nq::AttendLaunch L{};
  L.q = q;
  L.units = units;
  L.heads = heads;
  L.G = G;
  L.k_in = *k_in;
  L.v_in = *v_in;
  L.n = n;
  L.slot0 = slot0;
  L.positions = positions;
  L.pos_stride = pos_stride;
  L.pos_base = pos_base;
  L.rope_tab = rope_tab;
  L.rope_max_pos = rope_max_pos;
  L.scale = scale;
  L.out = out;
  L.lse = lse;
  L.ws = ws;
  return cuda_status(nq::launch_attend(L, reinterpret_cast<cudaStream_t>(stream)),
                     "nq_attend launch");
}

nq_status nq_e8_quantise(const float* y, int64_t groups, int bits, uint32_t* codes,
                         uint8_t* coset, nq_stream_t stream) {
  if (bits != 2 && bits != 3) return fail(NQ_ERR_INVALID, "bits must be 2 or 3 (got %d)", bits);
  if (groups < 0) return fail(NQ_ERR_INVALID, "groups must be >= 0");
  if (groups == 0) return NQ_OK;
  if (!y || !codes || !coset) return fail(NQ_ERR_INVALID, "y, codes and coset must be non-NULL");
  if (!aligned(y, 4) || !aligned(codes, 4))
    return fail(NQ_ERR_INVALID, "y and codes must be 4-byte aligned");
  return cuda_status(nq::launch_e8_quantise(y, groups, bits, codes, coset,
                                            reinterpret_cast<cudaStream_t>(stream)),
                     "nq_e8_quantise launch");
}

nq_status nq_e8_box_quantise(const float* y, int64_t groups, int bits, uint32_t* codes,
                             uint8_t* coset, nq_stream_t stream) {
  if (bits != 2 && bits != 3) return fail(NQ_ERR_INVALID, "bits must be 2 or 3 (got %d)", bits);
  if (groups < 0) return fail(NQ_ERR_INVALID, "groups must be >= 0");
  if (groups == 0) return NQ_OK;
  if (!y || !codes || !coset) return fail(NQ_ERR_INVALID, "y, codes and coset must be non-NULL");
  if (!aligned(y, 4) || !aligned(codes, 4))
    return fail(NQ_ERR_INVALID, "y and codes must be 4-byte aligned");
  return cuda_status(nq::launch_e8_box_quantise(y, groups, bits, codes, coset,
                                                reinterpret_cast<cudaStream_t>(stream)),
                     "nq_e8_box_quantise launch");
}

int64_t nq_entropy_streams(int units, int heads, int64_t n) {
  if (units < 0 || heads < 1 || n < 1) return 0;
  return nq::entropy_streams(units, heads, n);
}

int64_t nq_entropy_max_words(int units, int heads, int64_t n) {
  if (units < 0 || heads < 1 || n < 1) return 0;
  return nq::entropy_max_words(units, heads, n);
}

size_t nq_entropy_workspace_bytes(int units, int heads, int64_t n) {
  if (units < 0 || heads < 1 || n < 1) return 0;
  return nq::entropy_workspace_bytes(units, heads, n);
}

static nq_status check_entropy_shape(int units, int heads, int64_t n, int64_t slot0, int delta) {
  if (units < 0 || heads < 1 || heads > 1024)
    return fail(NQ_ERR_INVALID, "need units >= 0 and 1 <= heads <= 1024");
  if (n < 1 || n >= (int64_t(1) << 25))
    return fail(NQ_ERR_INVALID, "need 1 <= n < 2^25 (got %lld)", static_cast<long long>(n));
  if (slot0 < 0) return fail(NQ_ERR_INVALID, "slot0 must be >= 0");
  if (delta != 0 && delta != 1) return fail(NQ_ERR_INVALID, "delta must be 0 or 1");
  if (nq::entropy_max_words(units, heads, n) > 0xFFFFFFFFll)
    return fail(NQ_ERR_UNSUPPORTED, "units * heads * n too large for 32-bit stream offsets");
  return NQ_OK;
}

nq_status nq_entropy_encode(const nq_packed* in, int units, int heads, int64_t n, int64_t slot0,
                            int delta, uint16_t* freq, uint32_t* offsets, uint16_t* words,
                            int64_t words_cap, void* ws, size_t ws_bytes, nq_stream_t stream) {
  if (nq_status st = check_entropy_shape(units, heads, n, slot0, delta)) return st;
  if (nq_status st = check_packed(in, "in")) return st;
  if (units == 0) return NQ_OK;
  if (!freq || !offsets || !words || !ws)
    return fail(NQ_ERR_INVALID, "freq, offsets, words and ws must be non-NULL");
  if (!aligned(freq, 2) || !aligned(offsets, 4) || !aligned(words, 2) || !aligned(ws, 16))
    return fail(NQ_ERR_INVALID, "freq/words 2-byte, offsets 4-byte, ws 16-byte aligned");
  if (words_cap < nq::entropy_max_words(units, heads, n))
    return fail(NQ_ERR_WORKSPACE, "words_cap %lld < nq_entropy_max_words %lld",
                static_cast<long long>(words_cap),
                static_cast<long long>(nq::entropy_max_words(units, heads, n)));
  const size_t need = nq::entropy_workspace_bytes(units, heads, n);
  if (ws_bytes < need)
    return fail(NQ_ERR_WORKSPACE, "entropy workspace too small: %zu < %zu", ws_bytes, need);
  return cuda_status(nq::launch_entropy_encode(*in, units, heads, n, slot0, delta, freq, offsets,
                                               words, ws, reinterpret_cast<cudaStream_t>(stream)),
                     "nq_entropy_encode launch");
}

nq_status nq_entropy_decode(const uint16_t* words, const uint32_t* offsets, const uint16_t* freq,
                            int units, int heads, int64_t n, int delta, const nq_packed* out,
                            int64_t slot0, nq_stream_t stream) {
  if (nq_status st = check_entropy_shape(units, heads, n, slot0, delta)) return st;
  if (nq_status st = check_packed(out, "out")) return st;
  if (units == 0) return NQ_OK;
  if (!freq || !offsets || !words)
    return fail(NQ_ERR_INVALID, "words, offsets and freq must be non-NULL");
  if (!aligned(freq, 2) || !aligned(offsets, 4) || !aligned(words, 2))
    return fail(NQ_ERR_INVALID, "freq/words 2-byte, offsets 4-byte aligned");
  return cuda_status(nq::launch_entropy_decode(words, offsets, freq, units, heads, n, delta, *out,
                                               slot0, reinterpret_cast<cudaStream_t>(stream)),
                     "nq_entropy_decode launch");
}

nq_status nq_set_decode_engine(int engine) {
  if (engine != NQ_DECODE_AUTO && engine != NQ_DECODE_TENSOR_CORES && engine != NQ_DECODE_CUDA_CORES)
    return fail(NQ_ERR_INVALID, "decode engine must be 0, 1 or 2 (got %d)", engine);
  nq::set_decode_engine(engine);
  return NQ_OK;
}

int nq_get_decode_engine(void) { return nq::decode_engine(); }

nq_status nq_device_error(uint32_t* flags_out) {
  if (!flags_out) return fail(NQ_ERR_INVALID, "flags_out is NULL");
  return cuda_status(nq::codec_read_clear_error(flags_out), "nq_device_error");
}

}  // extern "C"
