// C ABI of libsol (declared in include/sol.h): host-side argument checks,
// then one kernel launch on the caller's stream.  Nothing is allocated and
// nothing is synchronised.
#include <algorithm>
#include <cstdarg>
#include <initializer_list>
#include <cstdio>
#include <map>
#include <mutex>
#include <string>
#include <tuple>

#include "sol.h"
#include "sol_launch.h"

namespace sol {
namespace {

thread_local std::string g_last_error;

sol_status fail(sol_status s, const char *fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return s;
}

sol_status ok() {
  g_last_error.clear();
  return SOL_OK;
}

sol_status cuda_fail(cudaError_t e, const char *what) {
  return fail(SOL_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int esize_of(sol_dtype dt) { return dt == SOL_F32 ? 4 : 2; }

// Byte range [begin, end) touched by `rows` rows of `width` bytes, `ld`
// bytes apart, starting at p.
struct Span {
  uintptr_t begin, end;
};
Span span_of(const void *p, int64_t rows, int64_t ld, int64_t width) {
  uintptr_t b = reinterpret_cast<uintptr_t>(p);
  return Span{b, b + static_cast<uintptr_t>((rows - 1) * ld + width)};
}
bool spans_overlap(Span a, Span b) { return a.begin < b.end && b.begin < a.end; }

// True if the strided blocks A (base a, width wa) and B (base b, width wb),
// both `rows` rows with the same row pitch `ld`, share no byte.  With equal
// pitches, B's columns sit at offset c = (b - a) mod ld inside A's rows and
// the blocks are disjoint when wa <= c <= ld - wb.
bool strided_disjoint(const void *a, int64_t wa, const void *b, int64_t wb, int64_t rows,
                      int64_t lda, int64_t ldb) {
  if (!spans_overlap(span_of(a, rows, lda, wa), span_of(b, rows, ldb, wb))) return true;
  if (lda != ldb) return false;
  const int64_t off = static_cast<int64_t>(reinterpret_cast<intptr_t>(b) -
                                           reinterpret_cast<intptr_t>(a));
  int64_t c = off % lda;
  if (c < 0) c += lda;
  return wa <= c && c <= lda - wb;
}

// Identical or disjoint, for two contiguous [rows, width] tensors.
bool same_or_disjoint(const void *a, const void *b, int64_t bytes) {
  if (a == b) return true;
  return !spans_overlap(span_of(a, 1, 0, bytes), span_of(b, 1, 0, bytes));
}

struct DevCache {
  std::mutex mu;
  std::map<int, int> sms;
  std::map<std::tuple<const void *, int, int, size_t>, int> occ;
  std::map<std::pair<const void *, int>, bool> attr_set;
};
DevCache &cache() {
  static DevCache c;
  return c;
}

}  // namespace

int device_sms() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  DevCache &c = cache();
  std::lock_guard<std::mutex> lk(c.mu);
  auto it = c.sms.find(dev);
  if (it != c.sms.end()) return it->second;
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  c.sms[dev] = n;
  return n;
}

int resident_blocks(const void *kernel, int threads, size_t smem) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  DevCache &c = cache();
  std::lock_guard<std::mutex> lk(c.mu);
  auto key = std::make_tuple(kernel, dev, threads, smem);
  auto it = c.occ.find(key);
  if (it != c.occ.end()) return it->second;
  auto akey = std::make_pair(kernel, dev);
  if (!c.attr_set[akey]) {
    // allow dynamic shared memory up to the opt-in limit less the kernel's
    // static shared memory (the attribute counts only the dynamic part)
    int optin = 0;
    cudaFuncAttributes fa{};
    if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) !=
            cudaSuccess ||
        cudaFuncGetAttributes(&fa, kernel) != cudaSuccess)
      return 0;
    const int dyn_max = optin - static_cast<int>(fa.sharedSizeBytes);
    if (dyn_max <= 0 ||
        cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn_max) !=
            cudaSuccess)
      return 0;
    c.attr_set[akey] = true;
  }
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, threads, smem) != cudaSuccess)
    return 0;
  c.occ[key] = n;
  return n;
}

bool pick_split(int64_t nvec, int *threads, int *vpt) {
  if (nvec <= 0) return false;
  for (int t = 32; t <= kMaxThreads; t *= 2) {
    const int64_t v = (nvec + t - 1) / t;
    if (v <= 6 || (t == kMaxThreads && v <= kMaxVpt)) {
      *threads = t;
      *vpt = static_cast<int>(v);
      return true;
    }
  }
  return false;
}

bool pick_split_qk(int64_t nvec, int *threads, int *vpt) {
  if (nvec <= 0) return false;
  for (int t = 32; t <= kMaxThreads; t *= 2) {
    const int64_t v = (nvec + t - 1) / t;
    if (v <= 3 || (t == kMaxThreads && v <= kMaxVpt)) {
      *threads = t;
      *vpt = static_cast<int>(v);
      return true;
    }
  }
  return false;
}

bool pick_split_otf(int64_t nvec, int *threads, int *vpt) {
  if (nvec <= 0 || nvec > 256 * kMaxVpt) return false;
  if (nvec <= 128) {
    *threads = 32;
    *vpt = static_cast<int>((nvec + 31) / 32);
  } else if (nvec <= 1024) {
    *threads = static_cast<int>(((nvec + 3) / 4 + 31) / 32 * 32);
    *vpt = 4;
  } else {
    *threads = 256;
    *vpt = static_cast<int>((nvec + 255) / 256);
  }
  return true;
}

bool pick_split_tab(int64_t nvec, int *threads, int *vpt) {
  static const int sizes[] = {32, 64, 96, 128, 160, 192, 224, 256, 320, 384, 448, 512};
  if (nvec <= 0 || nvec > 256 * kMaxVpt) return false;
  if (nvec <= 32) {
    *threads = 32;
    *vpt = 1;
  } else if (nvec <= 1024) {
    const int64_t half = (nvec + 1) / 2;
    int t = 512;
    for (int c : sizes)
      if (c >= half) {
        t = c;
        break;
      }
    *threads = t;
    *vpt = 2;
  } else {
    *threads = 256;
    *vpt = static_cast<int>((nvec + 255) / 256);
  }
  return true;
}

bool pick_split_i8w(int64_t slots, int *threads, int *vpt) {
  for (int t = 32; t <= 256; t *= 2) {
    const int64_t v = (slots + t - 1) / t;
    if (slots > 0 && v <= 5) {
      *threads = t;
      *vpt = static_cast<int>(v);
      return true;
    }
  }
  return false;
}

}  // namespace sol

namespace sol {
namespace {

// Argument checks of sol_qknorm_rope3d (and of its table-driven form, which
// passes the table's head_dim, sections and theta).  On SOL_OK either
// `empty` is set (zero rows: nothing to launch) or `a` is filled.
sol_status check_qk(const char *fn, const void *qkv, int64_t ld_qkv, void *q_out, void *k_out,
                    int64_t ld_out, const void *gamma_q, const void *gamma_k, int64_t B,
                    int64_t T, int64_t H, int64_t W, int64_t n_audio, int64_t n_heads,
                    int64_t head_dim, int64_t sec_t, int64_t sec_h, int64_t sec_w, float eps,
                    float theta, sol_dtype dtype, QkArgs &a, bool &empty) {
  empty = false;
  if (dtype != SOL_F32 && dtype != SOL_BF16)
    return fail(SOL_ERR_INVALID_ARG, "%s: unknown dtype %d", fn, (int)dtype);
  if (B < 0 || T < 0 || H < 0 || W < 0 || n_audio < 0)
    return fail(SOL_ERR_INVALID_ARG, "%s: B, T, H, W, n_audio must be >= 0", fn);
  if (n_heads <= 0 || head_dim <= 0 || head_dim % 2 != 0)
    return fail(SOL_ERR_INVALID_ARG, "%s: need n_heads > 0 and an even head_dim > 0 (%lld, %lld)",
                fn, (long long)n_heads, (long long)head_dim);
  if (sec_t < 0 || sec_h < 0 || sec_w < 0 || sec_t + sec_h + sec_w != head_dim / 2)
    return fail(SOL_ERR_INVALID_ARG, "%s: sections %lld+%lld+%lld must sum to head_dim/2 = %lld",
                fn, (long long)sec_t, (long long)sec_h, (long long)sec_w,
                (long long)(head_dim / 2));
  if (!(eps >= 0.f) || !(theta > 0.f))
    return fail(SOL_ERR_INVALID_ARG, "%s: need eps >= 0 and theta > 0", fn);
  if (T > kMaxRows || H > kMaxRows || W > kMaxRows || n_audio > kMaxRows || B > kMaxRows ||
      H * W > kMaxRows || T * H * W > kMaxRows || T * H * W + n_audio > kMaxRows ||
      B * (T * H * W + n_audio) > kMaxRows)
    return fail(SOL_ERR_UNSUPPORTED, "%s: B*L and H*W must be below 2^31", fn);
  const int64_t n_video = T * H * W;
  const int64_t L = n_video + n_audio;
  const int64_t rows = B * L;
  const int64_t D = n_heads * head_dim;
  if (ld_qkv < 2 * D || ld_out < D)
    return fail(SOL_ERR_INVALID_ARG, "%s: need ld_qkv >= 2*D and ld_out >= D", fn);
  if (rows == 0) {
    empty = true;
    return ok();
  }
  if (!qkv || !q_out || !k_out)
    return fail(SOL_ERR_INVALID_ARG, "%s: qkv, q_out and k_out must be non-null", fn);
  const int es = esize_of(dtype);
  const int64_t hd_bytes = head_dim * es;
  const int64_t G = hd_bytes / 16;
  if (hd_bytes % 16 != 0 || G < 2 || G > 32 || (G & (G - 1)) != 0)
    return fail(SOL_ERR_UNSUPPORTED,
                "%s: head_dim*%d bytes must be 16*G with G a power of two in "
                "[2, 32] (head_dim=%lld)",
                fn, es, (long long)head_dim);
  const int64_t ldq_b = ld_qkv * es, ldo_b = ld_out * es, D_b = D * es;
  if (!aligned16(qkv) || !aligned16(q_out) || !aligned16(k_out) || ldq_b % 16 || ldo_b % 16 ||
      (gamma_q && !aligned16(gamma_q)) || (gamma_k && !aligned16(gamma_k)))
    return fail(SOL_ERR_MISALIGNED, "%s: pointers and row strides must be 16-byte aligned", fn);
  if (2 * D_b > kMaxRowBytesQk)
    return fail(SOL_ERR_UNSUPPORTED, "%s: 2*D=%lld exceeds %lld elements", fn,
                (long long)(2 * D), (long long)(kMaxRowBytesQk / es));
  const bool in_place = q_out == qkv && ld_out == ld_qkv &&
                        static_cast<const unsigned char *>(k_out) ==
                            static_cast<const unsigned char *>(qkv) + D_b;
  if (!in_place) {
    if (!strided_disjoint(qkv, 2 * D_b, q_out, D_b, rows, ldq_b, ldo_b) ||
        !strided_disjoint(qkv, 2 * D_b, k_out, D_b, rows, ldq_b, ldo_b) ||
        !strided_disjoint(q_out, D_b, k_out, D_b, rows, ldo_b, ldo_b))
      return fail(SOL_ERR_INVALID_ARG,
                  "%s: outputs must be exactly in place (q_out=qkv, "
                  "k_out=qkv+D, ld_out=ld_qkv) or overlap neither qkv nor each other",
                  fn);
  }
  for (const void *g : {gamma_q, gamma_k}) {
    if (!g) continue;
    Span gs = span_of(g, 1, 0, hd_bytes);
    if (spans_overlap(gs, span_of(q_out, rows, ldo_b, D_b)) ||
        spans_overlap(gs, span_of(k_out, rows, ldo_b, D_b)))
      return fail(SOL_ERR_INVALID_ARG, "%s: an output overlaps gamma", fn);
  }

  a = QkArgs{};
  a.qkv = qkv;
  a.q_out = q_out;
  a.k_out = k_out;
  a.gamma_q = gamma_q;
  a.gamma_k = gamma_k;
  a.ld_qkv_bytes = ldq_b;
  a.ld_out_bytes = ldo_b;
  a.rows = rows;
  a.L = static_cast<int>(L);
  a.n_video = static_cast<int>(n_video);
  a.HW = static_cast<int>(H * W);
  a.H = static_cast<int>(H);
  a.W = static_cast<int>(W);
  a.nvec_q = static_cast<int>(D_b / 16);
  a.npairs = static_cast<int>(head_dim / 2);
  a.sec_t = static_cast<int>(sec_t);
  a.sec_th = static_cast<int>(sec_t + sec_h);
  a.head_dim = static_cast<int>(head_dim);
  a.eps = eps;
  a.inv_hd = static_cast<float>(1.0 / static_cast<double>(head_dim));
  a.theta = theta;
  return ok();
}

// The descriptor of a rotary table: fields in range, data aligned.
sol_status check_table(const char *fn, const sol_rope_table *tab) {
  if (!tab) return fail(SOL_ERR_INVALID_ARG, "%s: the table descriptor must be non-null", fn);
  if (tab->n_pos < 0 || tab->n_pos > kMaxRows)
    return fail(SOL_ERR_INVALID_ARG, "%s: table n_pos must be in [0, 2^31)", fn);
  if (tab->head_dim < 2 || tab->head_dim % 2 != 0 || tab->head_dim > 2 * kMaxRotaryPairs)
    return fail(SOL_ERR_INVALID_ARG, "%s: table head_dim must be even and in [2, %lld]", fn,
                (long long)(2 * kMaxRotaryPairs));
  if (tab->sec_t < 0 || tab->sec_h < 0 || tab->sec_w < 0 ||
      tab->sec_t + tab->sec_h + tab->sec_w != tab->head_dim / 2)
    return fail(SOL_ERR_INVALID_ARG, "%s: table sections must sum to head_dim/2", fn);
  if (!(tab->theta > 0.f) || (tab->per_axis_freq != 0 && tab->per_axis_freq != 1))
    return fail(SOL_ERR_INVALID_ARG, "%s: table theta must be > 0 and per_axis_freq 0 or 1", fn);
  if (!tab->data) return fail(SOL_ERR_INVALID_ARG, "%s: table data must be non-null", fn);
  if (!aligned16(tab->data))
    return fail(SOL_ERR_MISALIGNED, "%s: table data must be 16-byte aligned", fn);
  return ok();
}

// A call's use of a table: every position it meets is a row, and no output
// span overlaps the table.
sol_status check_table_use(const char *fn, const sol_rope_table *tab, int64_t T, int64_t H,
                           int64_t W, int64_t n_audio, std::initializer_list<Span> outs) {
  int64_t need = n_audio;
  if (T * H * W > 0) need = std::max(need, std::max(T, std::max(H, W)));
  if (tab->n_pos < need)
    return fail(SOL_ERR_INVALID_ARG,
                "%s: the table has %lld positions, the call needs %lld (max of T, H, W, n_audio)",
                fn, (long long)tab->n_pos, (long long)need);
  const Span ts = span_of(tab->data, 1, 0, static_cast<int64_t>(tab->n_pos) * tab->head_dim * 4);
  for (const Span &o : outs)
    if (tab->n_pos > 0 && spans_overlap(o, ts))
      return fail(SOL_ERR_INVALID_ARG, "%s: an output overlaps the rotary table", fn);
  return ok();
}

// sol_qknorm_rope3d_ex and its table-driven form (tab non-null: head_dim,
// sections and theta are the table's, and the rotation reads it).
sol_status qk_ex(const char *fn, const void *qkv, int64_t ld_qkv, void *q_out, void *k_out,
                 const sol_qk_layout *layout, const void *gamma_q, const void *gamma_k,
                 const sol_rope_table *tab, int64_t B, int64_t T, int64_t H, int64_t W,
                 int64_t n_audio, int64_t n_heads, int64_t head_dim, int64_t sec_t,
                 int64_t sec_h, int64_t sec_w, float eps, float theta, sol_dtype dtype,
                 sol_stream_t stream) {
  if (!layout) return fail(SOL_ERR_INVALID_ARG, "%s: layout must be non-null", fn);
  if (dtype != SOL_BF16)
    return fail(SOL_ERR_UNSUPPORTED, "%s: bf16 input only", fn);
  if (B < 0 || T < 0 || H < 0 || W < 0 || n_audio < 0 || n_heads <= 0)
    return fail(SOL_ERR_INVALID_ARG, "%s: B, T, H, W, n_audio must be >= 0, n_heads > 0", fn);
  if (head_dim != 64 && head_dim != 128 && head_dim != 256)
    return fail(SOL_ERR_UNSUPPORTED, "%s: head_dim must be 64, 128 or 256 (got %lld)", fn,
                (long long)head_dim);
  if (sec_t < 0 || sec_h < 0 || sec_w < 0 || sec_t + sec_h + sec_w != head_dim / 2)
    return fail(SOL_ERR_INVALID_ARG, "%s: sections must sum to head_dim/2", fn);
  if (!(eps >= 0.f) || !(theta > 0.f))
    return fail(SOL_ERR_INVALID_ARG, "%s: need eps >= 0 and theta > 0", fn);
  if (layout->stride_b < 0 || layout->stride_row < 0 || layout->stride_head < 0)
    return fail(SOL_ERR_INVALID_ARG, "%s: strides must be >= 0", fn);
  if (T > kMaxRows || H > kMaxRows || W > kMaxRows || n_audio > kMaxRows || B > kMaxRows ||
      H * W > kMaxRows || T * H * W > kMaxRows || T * H * W + n_audio > kMaxRows ||
      B * (T * H * W + n_audio) > kMaxRows)
    return fail(SOL_ERR_UNSUPPORTED, "%s: B*L and H*W must be below 2^31", fn);
  const int64_t n_video = T * H * W;
  const int64_t L = n_video + n_audio;
  const int64_t rows = B * L;
  const int64_t D = n_heads * head_dim;
  if (ld_qkv < 2 * D) return fail(SOL_ERR_INVALID_ARG, "%s: need ld_qkv >= 2*D", fn);
  if (rows == 0) return ok();
  const bool int8 = layout->int8_out != 0;
  if (layout->reserved != 0 || (layout->per_axis_freq != 0 && layout->per_axis_freq != 1))
    return fail(SOL_ERR_INVALID_ARG, "%s: layout.reserved must be 0, per_axis_freq 0 or 1", fn);
  const bool quant_v = layout->v_out != nullptr;
  if (quant_v && !int8)
    return fail(SOL_ERR_UNSUPPORTED, "%s: v_out needs int8_out (v is only quantised)", fn);
  if (!qkv || !q_out || !k_out || (int8 && (!layout->q_scale || !layout->k_scale)) ||
      (quant_v && !layout->v_scale))
    return fail(SOL_ERR_INVALID_ARG, "%s: qkv, q_out, k_out (and scales) must be non-null", fn);
  if (quant_v && ld_qkv < 3 * D)
    return fail(SOL_ERR_INVALID_ARG, "%s: quantising v needs ld_qkv >= 3*D", fn);
  if (2 * D * 2 > kMaxRowBytesQk)
    return fail(SOL_ERR_UNSUPPORTED, "%s: 2*D=%lld exceeds %lld elements", fn, (long long)(2 * D),
                (long long)(kMaxRowBytesQk / 2));
  const int oes = int8 ? 1 : 2;     // output element size
  const int vb = int8 ? 8 : 16;     // output bytes per thread vector
  const int64_t sb = layout->stride_b * oes, sr = layout->stride_row * oes,
                sh = layout->stride_head * oes;
  if (!aligned16(qkv) || (ld_qkv * 2) % 16 || (gamma_q && !aligned16(gamma_q)) ||
      (gamma_k && !aligned16(gamma_k)) || reinterpret_cast<uintptr_t>(q_out) % vb ||
      reinterpret_cast<uintptr_t>(k_out) % vb || sb % vb || sr % vb || sh % vb ||
      (int8 && ((reinterpret_cast<uintptr_t>(layout->q_scale) & 3u) ||
                (reinterpret_cast<uintptr_t>(layout->k_scale) & 3u))) ||
      (quant_v && ((reinterpret_cast<uintptr_t>(layout->v_out) % vb) ||
                   (reinterpret_cast<uintptr_t>(layout->v_scale) & 3u))))
    return fail(SOL_ERR_MISALIGNED, "%s: pointers and strides must be aligned", fn);
  // byte extent of one output: last element + 1
  const int64_t ext = (B - 1) * sb + (L - 1) * sr + (n_heads - 1) * sh + head_dim * oes;
  const Span qs = span_of(q_out, 1, 0, ext), ks = span_of(k_out, 1, 0, ext);
  // the columns read: q and k, and v too when it is quantised
  const Span in = span_of(qkv, rows, ld_qkv * 2, (quant_v ? 3 : 2) * D * 2);
  // v's codes: the layout of q_out; an empty span when v is not quantised
  const Span vs = quant_v ? span_of(layout->v_out, 1, 0, ext) : Span{0, 0};
  if (spans_overlap(qs, in) || spans_overlap(ks, in) || spans_overlap(qs, ks) ||
      spans_overlap(vs, in) || spans_overlap(vs, qs) || spans_overlap(vs, ks))
    return fail(SOL_ERR_INVALID_ARG,
                "%s: q_out, k_out and v_out must overlap neither qkv nor each other", fn);
  if (int8) {
    const int64_t sc = rows * n_heads * 4;
    const Span a1 = span_of(layout->q_scale, 1, 0, sc), a2 = span_of(layout->k_scale, 1, 0, sc);
    const Span a3 = quant_v ? span_of(layout->v_scale, 1, 0, sc) : Span{0, 0};
    for (const Span &z : {a1, a2, a3})
      if (spans_overlap(z, qs) || spans_overlap(z, ks) || spans_overlap(z, vs) ||
          spans_overlap(z, in))
        return fail(SOL_ERR_INVALID_ARG, "%s: a scale array overlaps a tensor", fn);
    if (spans_overlap(a1, a2) || spans_overlap(a1, a3) || spans_overlap(a2, a3))
      return fail(SOL_ERR_INVALID_ARG, "%s: the scale arrays overlap", fn);
  }
  for (const void *g : {gamma_q, gamma_k}) {
    if (!g) continue;
    const Span gs = span_of(g, 1, 0, head_dim * 2);
    if (spans_overlap(gs, qs) || spans_overlap(gs, ks) || spans_overlap(gs, vs))
      return fail(SOL_ERR_INVALID_ARG, "%s: an output overlaps gamma", fn);
  }

  if (tab) {
    const int64_t sc = int8 ? rows * n_heads * 4 : 0;
    const Span z{0, 0};
    const sol_status st = check_table_use(
        fn, tab, T, H, W, n_audio,
        {qs, ks, vs, int8 ? span_of(layout->q_scale, 1, 0, sc) : z,
         int8 ? span_of(layout->k_scale, 1, 0, sc) : z,
         quant_v ? span_of(layout->v_scale, 1, 0, sc) : z});
    if (st != SOL_OK) return st;
  }

  QkArgs a{};
  a.qkv = qkv;
  a.q_out = q_out;
  a.k_out = k_out;
  a.gamma_q = gamma_q;
  a.gamma_k = gamma_k;
  a.ld_qkv_bytes = ld_qkv * 2;
  a.ld_out_bytes = 0;
  a.rows = rows;
  a.L = static_cast<int>(L);
  a.n_video = static_cast<int>(n_video);
  a.HW = static_cast<int>(H * W);
  a.H = static_cast<int>(H);
  a.W = static_cast<int>(W);
  a.nvec_q = static_cast<int>(D * 2 / 16);
  a.npairs = static_cast<int>(head_dim / 2);
  a.sec_t = static_cast<int>(sec_t);
  a.sec_th = static_cast<int>(sec_t + sec_h);
  a.head_dim = static_cast<int>(head_dim);
  a.eps = eps;
  a.inv_hd = static_cast<float>(1.0 / static_cast<double>(head_dim));
  a.theta = theta;
  a.out_sb = sb;
  a.out_sr = sr;
  a.out_sh = sh;
  a.q_scale = layout->q_scale;
  a.k_scale = layout->k_scale;
  a.n_heads = static_cast<int>(n_heads);
  a.per_axis = layout->per_axis_freq;
  a.rope_tab = tab ? tab->data : nullptr;
  const bool half = layout->half_split != 0;
  cudaError_t e;
  if (tab)
    e = int8 ? launch_qknorm_rope3d_ex_tab_int8out(a, half, stream, nullptr)
             : launch_qknorm_rope3d_ex_tab_bf16out(a, half, stream, nullptr);
  else
    e = int8 ? launch_qknorm_rope3d_ex_int8out(a, half, stream, nullptr)
             : launch_qknorm_rope3d_ex_bf16out(a, half, stream, nullptr);
  if (e != cudaSuccess) return cuda_fail(e, fn);
  if (quant_v) {
    QuantArgs v{};
    v.src = static_cast<const unsigned char *>(qkv) + 2 * D * 2;
    v.ld_src_bytes = ld_qkv * 2;
    v.out = layout->v_out;
    v.scale = layout->v_scale;
    v.out_sb = sb;
    v.out_sr = sr;
    v.out_sh = sh;
    v.rows = rows;
    v.L = static_cast<int>(L);
    v.nvec = static_cast<int>(D * 2 / 16);
    v.n_heads = static_cast<int>(n_heads);
    e = launch_quantize_heads_int8(v, static_cast<int>(head_dim), stream, nullptr);
    if (e != cudaSuccess) return cuda_fail(e, fn);
  }
  return ok();
}

}  // namespace

}  // namespace sol

using namespace sol;

extern "C" {

int sol_version(void) { return (2 << 16) | 1; }

const char *sol_status_string(sol_status s) {
  switch (s) {
    case SOL_OK: return "SOL_OK";
    case SOL_ERR_INVALID_ARG: return "SOL_ERR_INVALID_ARG";
    case SOL_ERR_MISALIGNED: return "SOL_ERR_MISALIGNED";
    case SOL_ERR_UNSUPPORTED: return "SOL_ERR_UNSUPPORTED";
    case SOL_ERR_CUDA: return "SOL_ERR_CUDA";
  }
  return "SOL_ERR_UNKNOWN";
}

const char *sol_last_error(void) { return g_last_error.c_str(); }

sol_status sol_rms_adaln(const void *x, void *y, const void *scale, const void *shift,
                         const void *gamma, int64_t B, int64_t L, int64_t n_video, int64_t D,
                         float eps, sol_dtype dtype, sol_stream_t stream) {
  if (dtype != SOL_F32 && dtype != SOL_BF16)
    return fail(SOL_ERR_INVALID_ARG, "sol_rms_adaln: unknown dtype %d", (int)dtype);
  if (B < 0 || L < 0 || D <= 0 || n_video < 0 || n_video > L)
    return fail(SOL_ERR_INVALID_ARG,
                "sol_rms_adaln: need B >= 0, L >= 0, D > 0, 0 <= n_video <= L "
                "(B=%lld L=%lld n_video=%lld D=%lld)",
                (long long)B, (long long)L, (long long)n_video, (long long)D);
  if (!(eps >= 0.f)) return fail(SOL_ERR_INVALID_ARG, "sol_rms_adaln: eps must be >= 0");
  if (B > kMaxRows || L > kMaxRows || B * L > kMaxRows)
    return fail(SOL_ERR_UNSUPPORTED, "sol_rms_adaln: B*L must be below 2^31 rows");
  const int64_t rows = B * L;
  if (rows == 0) return ok();
  if (!x || !y || !scale || !shift)
    return fail(SOL_ERR_INVALID_ARG, "sol_rms_adaln: x, y, scale and shift must be non-null");
  const int es = esize_of(dtype);
  const int64_t row_bytes = D * es;
  if (row_bytes % 16 != 0)
    return fail(SOL_ERR_MISALIGNED, "sol_rms_adaln: D*%d bytes must be a multiple of 16 (D=%lld)",
                es, (long long)D);
  if (!aligned16(x) || !aligned16(y) || !aligned16(scale) || !aligned16(shift) ||
      (gamma && !aligned16(gamma)))
    return fail(SOL_ERR_MISALIGNED, "sol_rms_adaln: every pointer must be 16-byte aligned");
  if (row_bytes > kMaxRowBytesRms)
    return fail(SOL_ERR_UNSUPPORTED, "sol_rms_adaln: D=%lld exceeds %lld elements", (long long)D,
                (long long)(kMaxRowBytesRms / es));
  const int64_t act = rows * row_bytes, mod = B * 2 * row_bytes;
  if (!same_or_disjoint(x, y, act))
    return fail(SOL_ERR_INVALID_ARG, "sol_rms_adaln: y must equal x or not overlap it");
  Span ys = span_of(y, 1, 0, act);
  if (spans_overlap(ys, span_of(scale, 1, 0, mod)) || spans_overlap(ys, span_of(shift, 1, 0, mod)) ||
      (gamma && spans_overlap(ys, span_of(gamma, 1, 0, row_bytes))))
    return fail(SOL_ERR_INVALID_ARG, "sol_rms_adaln: y overlaps scale, shift or gamma");

  RmsArgs a{};
  a.x = x;
  a.y = y;
  a.scale = scale;
  a.shift = shift;
  a.gamma = gamma;
  a.rows = rows;
  a.L = static_cast<int>(L);
  a.n_video = static_cast<int>(n_video);
  a.nvec = static_cast<int>(row_bytes / 16);
  a.eps = eps;
  a.inv_D = static_cast<float>(1.0 / static_cast<double>(D));
  cudaError_t e = launch_rms_adaln(a, dtype == SOL_F32 ? 0 : 1, stream, nullptr);
  if (e != cudaSuccess) return cuda_fail(e, "sol_rms_adaln launch");
  return ok();
}

sol_status sol_gate_residual(const void *h, const void *branch, const void *gate, void *out,
                             int64_t B, int64_t L, int64_t n_video, int64_t D, sol_dtype dtype,
                             sol_stream_t stream) {
  if (dtype != SOL_F32 && dtype != SOL_BF16)
    return fail(SOL_ERR_INVALID_ARG, "sol_gate_residual: unknown dtype %d", (int)dtype);
  if (B < 0 || L < 0 || D <= 0 || n_video < 0 || n_video > L)
    return fail(SOL_ERR_INVALID_ARG,
                "sol_gate_residual: need B >= 0, L >= 0, D > 0, 0 <= n_video <= L "
                "(B=%lld L=%lld n_video=%lld D=%lld)",
                (long long)B, (long long)L, (long long)n_video, (long long)D);
  if (B > kMaxRows || L > kMaxRows || B * L > kMaxRows)
    return fail(SOL_ERR_UNSUPPORTED, "sol_gate_residual: B*L must be below 2^31 rows");
  const int64_t rows = B * L;
  if (rows == 0) return ok();
  if (!h || !branch || !gate || !out)
    return fail(SOL_ERR_INVALID_ARG, "sol_gate_residual: h, branch, gate and out must be non-null");
  const int es = esize_of(dtype);
  const int64_t row_bytes = D * es;
  if (row_bytes % 16 != 0)
    return fail(SOL_ERR_MISALIGNED,
                "sol_gate_residual: D*%d bytes must be a multiple of 16 (D=%lld)", es,
                (long long)D);
  if (!aligned16(h) || !aligned16(branch) || !aligned16(gate) || !aligned16(out))
    return fail(SOL_ERR_MISALIGNED, "sol_gate_residual: every pointer must be 16-byte aligned");
  if (row_bytes > kMaxRowBytesGate)
    return fail(SOL_ERR_UNSUPPORTED, "sol_gate_residual: D=%lld exceeds %lld elements",
                (long long)D, (long long)(kMaxRowBytesGate / es));
  const int64_t act = rows * row_bytes, mod = B * 2 * row_bytes;
  if (!same_or_disjoint(out, h, act) || !same_or_disjoint(out, branch, act))
    return fail(SOL_ERR_INVALID_ARG,
                "sol_gate_residual: out must equal h or branch, or overlap neither");
  if (spans_overlap(span_of(out, 1, 0, act), span_of(gate, 1, 0, mod)))
    return fail(SOL_ERR_INVALID_ARG, "sol_gate_residual: out overlaps gate");

  GateArgs a{};
  a.h = h;
  a.branch = branch;
  a.gate = gate;
  a.out = out;
  a.rows = rows;
  a.L = static_cast<int>(L);
  a.n_video = static_cast<int>(n_video);
  a.nvec = static_cast<int>(row_bytes / 16);
  cudaError_t e = launch_gate_residual(a, dtype == SOL_F32 ? 0 : 1, stream, nullptr);
  if (e != cudaSuccess) return cuda_fail(e, "sol_gate_residual launch");
  return ok();
}

sol_status sol_gate_residual_rms_adaln(const void *h, const void *branch, const void *gate,
                                       void *h_out, void *y, const void *scale,
                                       const void *shift, const void *gamma, int64_t B, int64_t L,
                                       int64_t n_video, int64_t D, float eps, sol_dtype dtype,
                                       sol_stream_t stream) {
  const char *fn = "sol_gate_residual_rms_adaln";
  if (dtype != SOL_F32 && dtype != SOL_BF16)
    return fail(SOL_ERR_INVALID_ARG, "%s: unknown dtype %d", fn, (int)dtype);
  if (B < 0 || L < 0 || D <= 0 || n_video < 0 || n_video > L)
    return fail(SOL_ERR_INVALID_ARG,
                "%s: need B >= 0, L >= 0, D > 0, 0 <= n_video <= L "
                "(B=%lld L=%lld n_video=%lld D=%lld)",
                fn, (long long)B, (long long)L, (long long)n_video, (long long)D);
  if (!(eps >= 0.f)) return fail(SOL_ERR_INVALID_ARG, "%s: eps must be >= 0", fn);
  if (B > kMaxRows || L > kMaxRows || B * L > kMaxRows)
    return fail(SOL_ERR_UNSUPPORTED, "%s: B*L must be below 2^31 rows", fn);
  const int64_t rows = B * L;
  if (rows == 0) return ok();
  if (!h || !branch || !gate || !h_out || !y || !scale || !shift)
    return fail(SOL_ERR_INVALID_ARG,
                "%s: h, branch, gate, h_out, y, scale and shift must be non-null", fn);
  const int es = esize_of(dtype);
  const int64_t row_bytes = D * es;
  if (row_bytes % 16 != 0)
    return fail(SOL_ERR_MISALIGNED, "%s: D*%d bytes must be a multiple of 16 (D=%lld)", fn, es,
                (long long)D);
  if (!aligned16(h) || !aligned16(branch) || !aligned16(gate) || !aligned16(h_out) ||
      !aligned16(y) || !aligned16(scale) || !aligned16(shift) || (gamma && !aligned16(gamma)))
    return fail(SOL_ERR_MISALIGNED, "%s: every pointer must be 16-byte aligned", fn);
  if (row_bytes > kMaxRowBytesRms)
    return fail(SOL_ERR_UNSUPPORTED, "%s: D=%lld exceeds %lld elements", fn, (long long)D,
                (long long)(kMaxRowBytesRms / es));
  const int64_t act = rows * row_bytes, mod = B * 2 * row_bytes;
  const Span hs = span_of(h, 1, 0, act), bs = span_of(branch, 1, 0, act),
             hos = span_of(h_out, 1, 0, act), ys = span_of(y, 1, 0, act);
  if (!same_or_disjoint(h_out, h, act) || spans_overlap(hos, bs))
    return fail(SOL_ERR_INVALID_ARG, "%s: h_out must equal h or overlap neither h nor branch",
                fn);
  if (spans_overlap(ys, hs) || spans_overlap(ys, bs) || spans_overlap(ys, hos))
    return fail(SOL_ERR_INVALID_ARG, "%s: y must not overlap h, branch or h_out", fn);
  for (const Span &o : {hos, ys}) {
    if (spans_overlap(o, span_of(gate, 1, 0, mod)) || spans_overlap(o, span_of(scale, 1, 0, mod)) ||
        spans_overlap(o, span_of(shift, 1, 0, mod)) ||
        (gamma && spans_overlap(o, span_of(gamma, 1, 0, row_bytes))))
      return fail(SOL_ERR_INVALID_ARG, "%s: an output overlaps gate, scale, shift or gamma", fn);
  }

  RmsArgs a{};
  a.x = h;
  a.y = y;
  a.scale = scale;
  a.shift = shift;
  a.gamma = gamma;
  a.branch = branch;
  a.gate = gate;
  a.h_out = h_out;
  a.rows = rows;
  a.L = static_cast<int>(L);
  a.n_video = static_cast<int>(n_video);
  a.nvec = static_cast<int>(row_bytes / 16);
  a.eps = eps;
  a.inv_D = static_cast<float>(1.0 / static_cast<double>(D));
  cudaError_t e = launch_gate_residual_rms_adaln(a, dtype == SOL_F32 ? 0 : 1, stream, nullptr);
  if (e != cudaSuccess) return cuda_fail(e, "sol_gate_residual_rms_adaln launch");
  return ok();
}

sol_status sol_qknorm_rope3d_ex(const void *qkv, int64_t ld_qkv, void *q_out, void *k_out,
                                const sol_qk_layout *layout, const void *gamma_q,
                                const void *gamma_k, int64_t B, int64_t T, int64_t H, int64_t W,
                                int64_t n_audio, int64_t n_heads, int64_t head_dim, int64_t sec_t,
                                int64_t sec_h, int64_t sec_w, float eps, float theta,
                                sol_dtype dtype, sol_stream_t stream) {
  return qk_ex("sol_qknorm_rope3d_ex", qkv, ld_qkv, q_out, k_out, layout, gamma_q, gamma_k,
               nullptr, B, T, H, W, n_audio, n_heads, head_dim, sec_t, sec_h, sec_w, eps, theta,
               dtype, stream);
}

sol_status sol_qknorm_rope3d_ex_tab(const void *qkv, int64_t ld_qkv, void *q_out, void *k_out,
                                    const sol_qk_layout *layout, const void *gamma_q,
                                    const void *gamma_k, const sol_rope_table *tab, int64_t B,
                                    int64_t T, int64_t H, int64_t W, int64_t n_audio,
                                    int64_t n_heads, float eps, sol_dtype dtype,
                                    sol_stream_t stream) {
  const char *fn = "sol_qknorm_rope3d_ex_tab";
  sol_status st = check_table(fn, tab);
  if (st != SOL_OK) return st;
  if (layout && layout->per_axis_freq != tab->per_axis_freq)
    return fail(SOL_ERR_INVALID_ARG,
                "%s: layout.per_axis_freq (%d) differs from the table's (%d)", fn,
                (int)layout->per_axis_freq, (int)tab->per_axis_freq);
  return qk_ex(fn, qkv, ld_qkv, q_out, k_out, layout, gamma_q, gamma_k, tab, B, T, H, W,
               n_audio, n_heads, tab->head_dim, tab->sec_t, tab->sec_h, tab->sec_w, eps,
               tab->theta, dtype, stream);
}

size_t sol_gemm_gelu_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  if (M <= 0 || N <= 0 || K <= 0 || M > kMaxRows || N > kMaxRows || K > kMaxRows) return 0;
  GemmArgs g{nullptr, nullptr, nullptr, nullptr, M, N, K};
  return gemm_gelu_workspace_bytes(g);
}

sol_status sol_gemm_gelu(const void *A, const void *B, const void *bias, void *C, int64_t M,
                         int64_t N, int64_t K, void *workspace, size_t workspace_bytes,
                         sol_stream_t stream) {
  const char *fn = "sol_gemm_gelu";
  if (M < 0 || N <= 0 || K <= 0)
    return fail(SOL_ERR_INVALID_ARG, "%s: need M >= 0, N > 0, K > 0", fn);
  if (M > kMaxRows || N > kMaxRows || K > kMaxRows)
    return fail(SOL_ERR_UNSUPPORTED, "%s: M, N, K must be below 2^31", fn);
  if (M == 0) return ok();
  if (!A || !B || !C) return fail(SOL_ERR_INVALID_ARG, "%s: A, B and C must be non-null", fn);
  if (N % 8 || K % 8)
    return fail(SOL_ERR_MISALIGNED, "%s: N and K must be multiples of 8 (N=%lld K=%lld)", fn,
                (long long)N, (long long)K);
  if (!aligned16(A) || !aligned16(B) || !aligned16(C) || (bias && !aligned16(bias)))
    return fail(SOL_ERR_MISALIGNED, "%s: pointers must be 16-byte aligned", fn);
  const Span cs = span_of(C, 1, 0, M * N * 2);
  if (spans_overlap(cs, span_of(A, 1, 0, M * K * 2)) ||
      spans_overlap(cs, span_of(B, 1, 0, N * K * 2)) ||
      (bias && spans_overlap(cs, span_of(bias, 1, 0, N * 2))))
    return fail(SOL_ERR_INVALID_ARG, "%s: C must not overlap A, B or bias", fn);
  GemmArgs g{A, B, bias, C, M, N, K};
  const size_t need = gemm_gelu_workspace_bytes(g);
  if (need > 0 && (!workspace || workspace_bytes < need))
    return fail(SOL_ERR_INVALID_ARG, "%s: workspace needs %zu bytes", fn, need);
  if (gemm_gelu_check(g) != 0)
    return fail(SOL_ERR_UNSUPPORTED, "%s: the GEMM templates reject this problem", fn);
  cudaError_t e = launch_gemm_gelu(g, workspace, stream);
  if (e != cudaSuccess) return cuda_fail(e, "sol_gemm_gelu launch");
  return ok();
}

size_t sol_residual_change_workspace_bytes(int64_t B) {
  return B <= 0 ? 0 : static_cast<size_t>(B) * kMaxChangeCtas * 2 * sizeof(double);
}

sol_status sol_residual_change(const void *cur, const void *prev, void *prev_out, int64_t B,
                               int64_t L, int64_t D, double *out, void *workspace,
                               size_t workspace_bytes, sol_dtype dtype, sol_stream_t stream) {
  const char *fn = "sol_residual_change";
  if (dtype != SOL_F32 && dtype != SOL_BF16)
    return fail(SOL_ERR_INVALID_ARG, "%s: unknown dtype %d", fn, (int)dtype);
  if (B < 0 || L < 0 || D <= 0)
    return fail(SOL_ERR_INVALID_ARG, "%s: need B >= 0, L >= 0, D > 0", fn);
  if (B > 65535 || L > kMaxRows || B * L > kMaxRows)
    return fail(SOL_ERR_UNSUPPORTED, "%s: need B <= 65535 and B*L below 2^31 rows", fn);
  const int64_t rows = B * L;
  if (rows == 0) return ok();
  if (!cur || !prev || !out || !workspace)
    return fail(SOL_ERR_INVALID_ARG, "%s: cur, prev, out and workspace must be non-null", fn);
  const int es = esize_of(dtype);
  const int64_t row_bytes = D * es;
  if (row_bytes % 16 != 0)
    return fail(SOL_ERR_MISALIGNED, "%s: D*%d bytes must be a multiple of 16 (D=%lld)", fn, es,
                (long long)D);
  if (!aligned16(cur) || !aligned16(prev) || (prev_out && !aligned16(prev_out)) ||
      !aligned16(workspace) || (reinterpret_cast<uintptr_t>(out) & 7u))
    return fail(SOL_ERR_MISALIGNED,
                "%s: tensors and workspace must be 16-byte aligned, out 8-byte aligned", fn);
  if (row_bytes > kMaxRowBytesRms)
    return fail(SOL_ERR_UNSUPPORTED, "%s: D=%lld exceeds %lld elements", fn, (long long)D,
                (long long)(kMaxRowBytesRms / es));
  const size_t need = sol_residual_change_workspace_bytes(B);
  if (workspace_bytes < need)
    return fail(SOL_ERR_INVALID_ARG, "%s: workspace has %zu bytes, needs %zu", fn,
                workspace_bytes, need);
  const int64_t act = rows * row_bytes;
  const Span cs = span_of(cur, 1, 0, act), ps = span_of(prev, 1, 0, act);
  const Span os = span_of(out, 1, 0, (B + 1) * 3 * 8), ws = span_of(workspace, 1, 0, need);
  if (prev_out) {
    const Span pos = span_of(prev_out, 1, 0, act);
    if (!same_or_disjoint(prev_out, prev, act) || spans_overlap(pos, cs))
      return fail(SOL_ERR_INVALID_ARG, "%s: prev_out must equal prev or overlap neither input",
                  fn);
    if (spans_overlap(os, pos) || spans_overlap(ws, pos))
      return fail(SOL_ERR_INVALID_ARG, "%s: out or workspace overlaps prev_out", fn);
  }
  if (spans_overlap(os, cs) || spans_overlap(os, ps) || spans_overlap(ws, cs) ||
      spans_overlap(ws, ps) || spans_overlap(os, ws))
    return fail(SOL_ERR_INVALID_ARG, "%s: out and workspace must not overlap the tensors or "
                "each other", fn);

  ChangeArgs a{};
  a.cur = cur;
  a.prev = prev;
  a.prev_out = prev_out;
  a.out = out;
  a.partial = static_cast<double *>(workspace);
  a.B = static_cast<int>(B);
  a.L = static_cast<int>(L);
  a.nvec = static_cast<int>(row_bytes / 16);
  cudaError_t e = launch_residual_change(a, dtype == SOL_F32 ? 0 : 1, stream, nullptr);
  if (e != cudaSuccess) return cuda_fail(e, "sol_residual_change launch");
  return ok();
}

sol_status sol_residual_change_noalloc(const void *cur, const void *prev, void *prev_out,
                                       int64_t B, int64_t L, int64_t D, double *out,
                                       sol_dtype dtype, sol_stream_t stream) {
  const char *fn = "sol_residual_change_noalloc";
  if (dtype != SOL_F32 && dtype != SOL_BF16)
    return fail(SOL_ERR_INVALID_ARG, "%s: unknown dtype %d", fn, (int)dtype);
  if (B < 0 || L < 0 || D <= 0)
    return fail(SOL_ERR_INVALID_ARG, "%s: need B >= 0, L >= 0, D > 0", fn);
  if (B > kNoAllocMaxSamples)
    return fail(SOL_ERR_UNSUPPORTED,
                "%s: B=%lld exceeds the %d samples its built-in scratch holds; use "
                "sol_residual_change with a workspace",
                fn, (long long)B, kNoAllocMaxSamples);
  if (L > kMaxRows || B * L > kMaxRows)
    return fail(SOL_ERR_UNSUPPORTED, "%s: B*L must be below 2^31 rows", fn);
  const int64_t rows = B * L;
  if (rows == 0) return ok();
  if (!cur || !prev || !out)
    return fail(SOL_ERR_INVALID_ARG, "%s: cur, prev and out must be non-null", fn);
  const int es = esize_of(dtype);
  const int64_t row_bytes = D * es;
  if (row_bytes % 16 != 0)
    return fail(SOL_ERR_MISALIGNED, "%s: D*%d bytes must be a multiple of 16 (D=%lld)", fn, es,
                (long long)D);
  if (!aligned16(cur) || !aligned16(prev) || (prev_out && !aligned16(prev_out)) ||
      (reinterpret_cast<uintptr_t>(out) & 7u))
    return fail(SOL_ERR_MISALIGNED, "%s: tensors must be 16-byte aligned, out 8-byte aligned",
                fn);
  if (row_bytes > kMaxRowBytesRms)
    return fail(SOL_ERR_UNSUPPORTED, "%s: D=%lld exceeds %lld elements", fn, (long long)D,
                (long long)(kMaxRowBytesRms / es));
  const int64_t act = rows * row_bytes;
  const Span cs = span_of(cur, 1, 0, act), ps = span_of(prev, 1, 0, act);
  const Span os = span_of(out, 1, 0, (B + 1) * 3 * 8);
  if (prev_out) {
    const Span pos = span_of(prev_out, 1, 0, act);
    if (!same_or_disjoint(prev_out, prev, act) || spans_overlap(pos, cs))
      return fail(SOL_ERR_INVALID_ARG, "%s: prev_out must equal prev or overlap neither input",
                  fn);
    if (spans_overlap(os, pos))
      return fail(SOL_ERR_INVALID_ARG, "%s: out overlaps prev_out", fn);
  }
  if (spans_overlap(os, cs) || spans_overlap(os, ps))
    return fail(SOL_ERR_INVALID_ARG, "%s: out must not overlap cur or prev", fn);

  ChangeArgs a{};
  a.cur = cur;
  a.prev = prev;
  a.prev_out = prev_out;
  a.out = out;
  a.B = static_cast<int>(B);
  a.L = static_cast<int>(L);
  a.nvec = static_cast<int>(row_bytes / 16);
  cudaError_t e = launch_residual_change_noalloc(a, dtype == SOL_F32 ? 0 : 1, stream, nullptr);
  if (e != cudaSuccess) return cuda_fail(e, "sol_residual_change_noalloc launch");
  return ok();
}

sol_status sol_qknorm_rope3d(const void *qkv, int64_t ld_qkv, void *q_out, void *k_out,
                             int64_t ld_out, const void *gamma_q, const void *gamma_k, int64_t B,
                             int64_t T, int64_t H, int64_t W, int64_t n_audio, int64_t n_heads,
                             int64_t head_dim, int64_t sec_t, int64_t sec_h, int64_t sec_w,
                             float eps, float theta, sol_dtype dtype, sol_stream_t stream) {
  const char *fn = "sol_qknorm_rope3d";
  QkArgs a{};
  bool empty = false;
  sol_status st = check_qk(fn, qkv, ld_qkv, q_out, k_out, ld_out, gamma_q, gamma_k, B, T, H, W,
                           n_audio, n_heads, head_dim, sec_t, sec_h, sec_w, eps, theta, dtype, a,
                           empty);
  if (st != SOL_OK || empty) return st;
  cudaError_t e = launch_qknorm_rope3d(a, dtype == SOL_F32 ? 0 : 1, stream, nullptr);
  if (e != cudaSuccess) return cuda_fail(e, "sol_qknorm_rope3d launch");
  return ok();
}

size_t sol_rope_table_bytes(int64_t n_pos, int64_t head_dim) {
  if (n_pos < 0 || n_pos > kMaxRows || head_dim < 2 || head_dim > 2 * kMaxRotaryPairs ||
      head_dim % 2 != 0)
    return 0;
  return static_cast<size_t>(n_pos) * static_cast<size_t>(head_dim) * 4u;
}

sol_status sol_rope_table_build(const sol_rope_table *tab, sol_stream_t stream) {
  const char *fn = "sol_rope_table_build";
  sol_status st = check_table(fn, tab);
  if (st != SOL_OK) return st;
  if (tab->n_pos == 0) return ok();
  cudaError_t e = launch_rope_table(tab->data, static_cast<int>(tab->n_pos),
                                    static_cast<int>(tab->head_dim / 2),
                                    static_cast<int>(tab->head_dim), static_cast<int>(tab->sec_t),
                                    static_cast<int>(tab->sec_t + tab->sec_h), tab->theta,
                                    tab->per_axis_freq, stream);
  if (e != cudaSuccess) return cuda_fail(e, "sol_rope_table_build launch");
  return ok();
}

sol_status sol_qknorm_rope3d_tab(const void *qkv, int64_t ld_qkv, void *q_out, void *k_out,
                                 int64_t ld_out, const void *gamma_q, const void *gamma_k,
                                 const sol_rope_table *tab, int64_t B, int64_t T, int64_t H,
                                 int64_t W, int64_t n_audio, int64_t n_heads, float eps,
                                 sol_dtype dtype, sol_stream_t stream) {
  const char *fn = "sol_qknorm_rope3d_tab";
  sol_status st = check_table(fn, tab);
  if (st != SOL_OK) return st;
  QkArgs a{};
  bool empty = false;
  st = check_qk(fn, qkv, ld_qkv, q_out, k_out, ld_out, gamma_q, gamma_k, B, T, H, W, n_audio,
                n_heads, tab->head_dim, tab->sec_t, tab->sec_h, tab->sec_w, eps, tab->theta,
                dtype, a, empty);
  if (st != SOL_OK || empty) return st;
  const int es = esize_of(dtype);
  const int64_t D_b = n_heads * tab->head_dim * es;
  st = check_table_use(fn, tab, T, H, W, n_audio,
                       {span_of(q_out, a.rows, a.ld_out_bytes, D_b),
                        span_of(k_out, a.rows, a.ld_out_bytes, D_b)});
  if (st != SOL_OK) return st;
  a.rope_tab = tab->data;
  cudaError_t e = launch_qknorm_rope3d(a, dtype == SOL_F32 ? 0 : 1, stream, nullptr);
  if (e != cudaSuccess) return cuda_fail(e, "sol_qknorm_rope3d_tab launch");
  return ok();
}

}  // extern "C"
