// C ABI entry points: argument validation on the host, then one launch on the
// caller's stream. See include/gdn2.h for the contract of each call.

#include <atomic>
#include <cmath>
#include <cstdint>

#include "common.cuh"

using namespace gdn2;

namespace {

bool aligned16(const void* p) { return p == nullptr || (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool supported_dim(int d) { return d == 16 || d == 32 || d == 64 || d == 128; }

// Byte range [p, p + n) overlaps [q, q + m)?
bool overlaps(const void* p, size_t n, const void* q, size_t m) {
  if (!p || !q || n == 0 || m == 0) return false;
  const uintptr_t a = reinterpret_cast<uintptr_t>(p), b = reinterpret_cast<uintptr_t>(q);
  return a < b + m && b < a + n;
}

size_t dsize(int dtype) { return dtype == GDN2_BF16 ? 2 : 4; }

// Sequences that own a state: n_seqs for packed sequences of different lengths, else B.
size_t n_states(const gdn2_params* p) { return p->cu_seqlens ? (size_t)p->n_seqs : (size_t)p->B; }

// Packed sequences (cu_seqlens): one row of B, 1..GDN2_MAX_SEQS sequences whose
// host offsets start at 0, never decrease and end at T.
gdn2_status check_varlen(const gdn2_params* p, bool decode) {
  if (!p->cu_seqlens) return p->n_seqs == 0 ? GDN2_OK : GDN2_ERR_INVALID_ARG;
  if (decode) return GDN2_ERR_INVALID_ARG;
  if (p->B != 1 || p->n_seqs < 1 || p->n_seqs > GDN2_MAX_SEQS) return GDN2_ERR_INVALID_ARG;
  const int* cu = p->cu_seqlens;
  if (cu[0] != 0 || cu[p->n_seqs] != p->T) return GDN2_ERR_INVALID_ARG;
  for (int n = 0; n < p->n_seqs; ++n)
    if (cu[n + 1] < cu[n]) return GDN2_ERR_INVALID_ARG;
  return GDN2_OK;
}

// Shared shape/enum checks. tokens = B*T (chunk) or B (decode).
gdn2_status check_common(const gdn2_params* p, bool decode) {
  if (!p) return GDN2_ERR_INVALID_ARG;
  if (p->B < 0 || (!decode && p->T < 0) || p->H_qk <= 0 || p->H_v <= 0) return GDN2_ERR_INVALID_ARG;
  if (p->H_v % p->H_qk != 0) return GDN2_ERR_INVALID_ARG;
  if (p->d_k <= 0 || p->d_v <= 0) return GDN2_ERR_INVALID_ARG;
  if (p->qkv_dtype != GDN2_F32 && p->qkv_dtype != GDN2_BF16) return GDN2_ERR_INVALID_ARG;
  if (p->o_dtype != GDN2_F32 && p->o_dtype != GDN2_BF16) return GDN2_ERR_INVALID_ARG;
  if (p->gate_mode < GDN2_GATES_FULL || p->gate_mode > GDN2_GATES_GDN) return GDN2_ERR_INVALID_ARG;
  if (p->gate_logits != 0 && p->gate_logits != 1) return GDN2_ERR_INVALID_ARG;
  if (p->gate_heads != GDN2_GATE_HEADS_V && p->gate_heads != GDN2_GATE_HEADS_QK) return GDN2_ERR_INVALID_ARG;
  if (p->precision != GDN2_PREC_DEFAULT && p->precision != GDN2_PREC_FP32) return GDN2_ERR_INVALID_ARG;
  if (!std::isfinite(p->scale)) return GDN2_ERR_INVALID_ARG;
  if (check_varlen(p, decode) != GDN2_OK) return GDN2_ERR_INVALID_ARG;
  if (p->d_k != p->d_v || !supported_dim(p->d_k)) return GDN2_ERR_UNSUPPORTED;
  // Element counts must fit comfortably in 63 bits and grid sizes in 31.
  const double elems = (double)p->B * (decode ? 1.0 : (double)p->T) * p->H_v * p->d_k;
  if (elems > 9.0e15) return GDN2_ERR_INVALID_ARG;
  if ((double)p->B * p->H_v * (p->d_k / 16) > 2.0e9) return GDN2_ERR_INVALID_ARG;
  return GDN2_OK;
}

struct Sizes {
  size_t qk, v, ga, gb, gw, st;  // bytes of q (= k), v, alpha, b, w, state
};

Sizes sizes(const gdn2_params* p, size_t tokens) {
  Sizes s;
  const size_t dk = p->d_k, dv = p->d_v;
  s.qk = tokens * p->H_qk * dk * dsize(p->qkv_dtype);
  s.v = tokens * p->H_v * dv * dsize(p->qkv_dtype);
  const size_t gsz = p->gate_logits ? 2 : 4;   // bf16 logits or fp32 values
  const size_t hg = p->gate_heads == GDN2_GATE_HEADS_QK ? p->H_qk : p->H_v;   // heads of alpha and b
  s.ga = tokens * hg * (p->gate_mode == GDN2_GATES_GDN ? 1 : dk) * gsz;
  s.gb = tokens * hg * (p->gate_mode == GDN2_GATES_FULL ? dk : 1) * gsz;
  s.gw = p->gate_mode == GDN2_GATES_FULL ? tokens * p->H_v * dv * gsz : 0;
  s.st = n_states(p) * p->H_v * dk * dv * 4;
  return s;
}

gdn2_status check_gate_ptrs(const gdn2_params* p, const float* alpha, const float* b, const float* w) {
  if (!alpha || !b) return GDN2_ERR_INVALID_ARG;
  if (p->gate_mode == GDN2_GATES_FULL ? (w == nullptr) : (w != nullptr)) return GDN2_ERR_INVALID_ARG;
  return GDN2_OK;
}

// Conv history buffers: only with a conv, 16-byte aligned; the outgoing
// history overlaps nothing else of the call, and no output overlaps the
// incoming history. `ins` / `outs` are the call's other inputs / outputs.
struct Range { const void* p; size_t n; };
gdn2_status check_conv_state(const gdn2_params* p, const Range* ins, int n_in, const Range* outs, int n_out) {
  const void* hin = p->conv_state_in;
  void* hout = p->conv_state_out;
  if (!p->conv_w && (hin || hout)) return GDN2_ERR_INVALID_ARG;
  if (!aligned16(hin) || !aligned16(hout)) return GDN2_ERR_INVALID_ARG;
  const size_t hb = n_states(p) * 3 * ((size_t)2 * p->H_qk * p->d_k + (size_t)p->H_v * p->d_v) *
                    dsize(p->qkv_dtype);
  if (overlaps(hout, hb, hin, hb)) return GDN2_ERR_INVALID_ARG;
  for (int i = 0; i < n_in; ++i)
    if (overlaps(hout, hb, ins[i].p, ins[i].n)) return GDN2_ERR_INVALID_ARG;
  for (int i = 0; i < n_out; ++i)
    if (overlaps(hout, hb, outs[i].p, outs[i].n) || overlaps(hin, hb, outs[i].p, outs[i].n))
      return GDN2_ERR_INVALID_ARG;
  return GDN2_OK;
}

ChunkArgs make_chunk_args(const gdn2_params* p, const void* q, const void* k, const void* v,
                          const float* alpha, const float* b, const float* w, const float* S0, void* o,
                          float* S_T, void* ws, size_t ws_bytes) {
  ChunkArgs a;
  a.B = p->B; a.T = p->T; a.Hqk = p->H_qk; a.Hv = p->H_v; a.dk = p->d_k; a.dv = p->d_v;
  a.chunk = p->chunk; a.scale = p->scale; a.gate_mode = p->gate_mode; a.l2norm = p->l2norm_qk != 0;
  a.conv_w = p->conv_w;
  a.gate_logits = p->gate_logits;
  a.conv_in = p->conv_state_in;
  a.conv_out = p->conv_state_out;
  a.Hg = p->gate_heads == GDN2_GATE_HEADS_QK ? p->H_qk : p->H_v;
  a.nseq = 0;
  if (p->cu_seqlens) {
    // B becomes the number of sequences; the 64-token chunks of the
    // tensor-core prefill start anew in every sequence.
    a.nseq = p->n_seqs;
    a.B = p->n_seqs;
    a.cu_chk[0] = 0;
    for (int n = 0; n <= p->n_seqs; ++n) a.cu_tok[n] = p->cu_seqlens[n];
    for (int n = 0; n < p->n_seqs; ++n) a.cu_chk[n + 1] = a.cu_chk[n] + (a.cu_tok[n + 1] - a.cu_tok[n] + 63) / 64;
  }
  a.q = q; a.k = k; a.v = v; a.alpha = alpha; a.b = b; a.w = w; a.S0 = S0; a.o = o; a.ST = S_T;
  a.workspace = ws; a.ws_bytes = ws_bytes;
  a.stall_polls = 0;
  return a;
}

std::atomic<unsigned> g_scan_stall{0};

bool use_tc(const gdn2_params* p, const ChunkArgs& a) {
  return p->precision == GDN2_PREC_DEFAULT && p->T > 0 && p->B > 0 &&
         chunk_tc_supported(a, p->qkv_dtype == GDN2_BF16);
}

}  // namespace

gdn2_status gdn2::check_chunk_params(const gdn2_params* p) {
  const gdn2_status st = check_common(p, false);
  if (st != GDN2_OK) return st;
  if (p->chunk != 16 && p->chunk != 32 && p->chunk != 64) return GDN2_ERR_UNSUPPORTED;
  return GDN2_OK;
}

unsigned gdn2::scan_stall_polls() { return g_scan_stall.load(std::memory_order_relaxed); }

gdn2_status gdn2::read_device_status(const void* scratch, cudaStream_t stream) {
  int word = 0;
  if (cudaMemcpyAsync(&word, scratch, sizeof(word), cudaMemcpyDeviceToHost, stream) != cudaSuccess ||
      cudaStreamSynchronize(stream) != cudaSuccess)
    return GDN2_ERR_CUDA;
  return word == 0 ? GDN2_OK : GDN2_ERR_TIMEOUT;
}

gdn2_status gdn2::chunk_fwd_checked(const gdn2_params* p, const void* q, const void* k, const void* v,
                                     const float* alpha, const float* b, const float* w, const float* S0,
                                     void* o, float* S_T, void* workspace, size_t ws_bytes, void* stream,
                                     bool segmented_ok) {
  gdn2_status st = check_chunk_params(p);
  if (st != GDN2_OK) return st;
  const size_t tokens = (size_t)p->B * p->T;
  if (tokens > 0) {
    if (!q || !k || !v || !o) return GDN2_ERR_INVALID_ARG;
    if ((st = check_gate_ptrs(p, alpha, b, w)) != GDN2_OK) return st;
  }
  const void* ptrs[] = {q, k, v, alpha, b, w, S0, o, S_T, p->conv_w, workspace};
  for (const void* ptr : ptrs)
    if (!aligned16(ptr)) return GDN2_ERR_INVALID_ARG;
  const Sizes sz = sizes(p, tokens);
  const size_t o_bytes = tokens * p->H_v * p->d_v * dsize(p->o_dtype);
  const size_t conv_bytes = ((size_t)2 * p->H_qk * p->d_k + (size_t)p->H_v * p->d_v) * 4 * sizeof(float);
  struct R { const void* p; size_t n; } ins[] = {{q, sz.qk}, {k, sz.qk}, {v, sz.v}, {alpha, sz.ga},
                                                  {b, sz.gb}, {w, sz.gw}, {S0, sz.st}, {p->conv_w, conv_bytes}};
  for (const R& r : ins) {
    if (overlaps(o, o_bytes, r.p, r.n)) return GDN2_ERR_INVALID_ARG;
    if (r.p != S0 && overlaps(S_T, sz.st, r.p, r.n)) return GDN2_ERR_INVALID_ARG;
  }
  if (S0 && S_T && S0 != S_T && overlaps(S0, sz.st, S_T, sz.st)) return GDN2_ERR_INVALID_ARG;
  if (overlaps(o, o_bytes, S_T, sz.st)) return GDN2_ERR_INVALID_ARG;
  {
    const Range cin[] = {{q, sz.qk}, {k, sz.qk}, {v, sz.v}, {alpha, sz.ga}, {b, sz.gb},
                         {w, sz.gw}, {S0, sz.st}, {p->conv_w, conv_bytes}};
    const Range cout[] = {{o, o_bytes}, {S_T, sz.st}, {workspace, ws_bytes}};
    if ((st = check_conv_state(p, cin, 8, cout, 3)) != GDN2_OK) return st;
  }

  ChunkArgs a = make_chunk_args(p, q, k, v, alpha, b, w, S0, o, S_T, workspace, ws_bytes);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (use_tc(p, a)) {
    const size_t need = segmented_ok ? chunk_tc_min_workspace(a, S_T == nullptr) : chunk_tc_workspace(a);
    if (need > 0 && (workspace == nullptr || ws_bytes < need)) return GDN2_ERR_WORKSPACE;
    if (workspace && (reinterpret_cast<uintptr_t>(workspace) & 255u)) return GDN2_ERR_INVALID_ARG;
    if (need > 0 && (overlaps(workspace, ws_bytes, o, o_bytes) || overlaps(workspace, ws_bytes, S_T, sz.st)))
      return GDN2_ERR_INVALID_ARG;
    a.ws_bytes = segmented_ok ? ws_bytes : chunk_tc_workspace(a);
    a.stall_polls = scan_stall_polls();
    e = launch_chunk_tc(a, p->o_dtype == GDN2_BF16, s);
  } else {
    e = launch_chunk_simt(a, p->qkv_dtype == GDN2_BF16, p->o_dtype == GDN2_BF16, s);
  }
  if (e == cudaSuccess) e = launch_conv_state(a, p->qkv_dtype == GDN2_BF16, s);
  return e == cudaSuccess ? GDN2_OK : GDN2_ERR_CUDA;
}

extern "C" {

const char* gdn2_status_str(gdn2_status s) {
  switch (s) {
    case GDN2_OK: return "GDN2_OK";
    case GDN2_ERR_INVALID_ARG: return "GDN2_ERR_INVALID_ARG: invalid argument (pointer, shape, alignment or aliasing)";
    case GDN2_ERR_UNSUPPORTED: return "GDN2_ERR_UNSUPPORTED: no kernel for this configuration";
    case GDN2_ERR_WORKSPACE: return "GDN2_ERR_WORKSPACE: workspace missing or too small";
    case GDN2_ERR_CUDA: return "GDN2_ERR_CUDA: CUDA launch or runtime error";
    case GDN2_ERR_TIMEOUT: return "GDN2_ERR_TIMEOUT: a device-side wait gave up";
  }
  return "GDN2: unknown status";
}

int gdn2_version(void) { return 200; }   // 0.2.0: gdn2_params grew the gate, conv-history and packed-sequence fields

size_t gdn2_chunk_fwd_workspace(const gdn2_params* p) {
  if (check_common(p, false) != GDN2_OK) return 0;
  ChunkArgs a = make_chunk_args(p, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr,
                                nullptr, nullptr, 0);
  return use_tc(p, a) ? chunk_tc_workspace(a) : 0;
}

gdn2_status gdn2_chunk_fwd(const gdn2_params* p, const void* q, const void* k, const void* v,
                           const float* alpha, const float* b, const float* w, const float* S0, void* o,
                           float* S_T, void* workspace, size_t ws_bytes, void* stream) {
  return gdn2::chunk_fwd_checked(p, q, k, v, alpha, b, w, S0, o, S_T, workspace, ws_bytes, stream, false);
}

gdn2_status gdn2_state_affine(const gdn2_params* p, const float* M, const float* N, const float* S_in,
                              float* S_out, void* stream) {
  if (!p || p->B < 0 || p->H_v <= 0 || p->d_k <= 0 || p->d_v <= 0) return GDN2_ERR_INVALID_ARG;
  if (p->d_k != p->d_v || !supported_dim(p->d_k) || p->d_k < 32) return GDN2_ERR_UNSUPPORTED;
  const size_t n = (size_t)p->B * p->H_v;
  if (n == 0) return GDN2_OK;
  if (!M || !S_out) return GDN2_ERR_INVALID_ARG;
  const void* ptrs[] = {M, N, S_in, S_out};
  for (const void* ptr : ptrs)
    if (!aligned16(ptr)) return GDN2_ERR_INVALID_ARG;
  const size_t sb = n * p->d_k * p->d_v * sizeof(float), mb = n * p->d_k * p->d_k * sizeof(float);
  // S_out may be S_in; nothing else overlaps it
  if (overlaps(S_out, sb, M, mb) || overlaps(S_out, sb, N, sb)) return GDN2_ERR_INVALID_ARG;
  if (S_in && S_in != S_out && overlaps(S_out, sb, S_in, sb)) return GDN2_ERR_INVALID_ARG;
  const cudaError_t e = launch_state_affine((int)n, p->d_k, p->d_v, M, N, S_in, S_out, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? GDN2_OK : GDN2_ERR_CUDA;
}

gdn2_status gdn2_chunk_fwd_status(const void* workspace, void* stream) {
  if (workspace == nullptr) return GDN2_OK;   // the fp32 path keeps no device status
  if (reinterpret_cast<uintptr_t>(workspace) & 255u) return GDN2_ERR_INVALID_ARG;
  return gdn2::read_device_status(workspace, static_cast<cudaStream_t>(stream));
}

void gdn2_debug_set_scan_stall(unsigned polls) { g_scan_stall.store(polls, std::memory_order_relaxed); }

size_t gdn2_chunk_bwd_workspace(const gdn2_params* p) {
  if (check_chunk_params(p) != GDN2_OK || p->conv_w || p->l2norm_qk || p->cu_seqlens) return 0;
  return chunk_bwd_workspace(p->B, p->H_v, p->T, p->d_k);
}

gdn2_status gdn2_chunk_bwd(const gdn2_params* p, const void* q, const void* k, const void* v,
                           const float* alpha, const float* b, const float* w, const float* S0, const void* dO,
                           const float* dS_T, float* dq, float* dk, float* dv, float* dalpha, float* db, float* dw,
                           float* dS0, void* workspace, size_t ws_bytes, void* stream) {
  gdn2_status st = check_chunk_params(p);
  if (st != GDN2_OK) return st;
  // the fused conv / L2 norm and packed sequences have no backward here
  if (p->conv_w || p->l2norm_qk || p->cu_seqlens || p->conv_state_in || p->conv_state_out)
    return GDN2_ERR_UNSUPPORTED;
  const size_t tokens = (size_t)p->B * p->T;
  const bool full = p->gate_mode == GDN2_GATES_FULL;
  if (tokens > 0) {
    if (!q || !k || !v || !dO || !dq || !dk || !dv || !dalpha || !db) return GDN2_ERR_INVALID_ARG;
    if ((st = check_gate_ptrs(p, alpha, b, w)) != GDN2_OK) return st;
    if (full ? dw == nullptr : dw != nullptr) return GDN2_ERR_INVALID_ARG;
  }
  const void* ptrs[] = {q, k, v, alpha, b, w, S0, dO, dS_T, dq, dk, dv, dalpha, db, dw, dS0, workspace};
  for (const void* ptr : ptrs)
    if (!aligned16(ptr)) return GDN2_ERR_INVALID_ARG;
  const Sizes sz = sizes(p, tokens);
  const size_t do_bytes = tokens * p->H_v * p->d_v * dsize(p->o_dtype);
  const size_t f32 = sizeof(float);
  const size_t ga32 = sz.ga / (p->gate_logits ? 2 : 4) * f32, gb32 = sz.gb / (p->gate_logits ? 2 : 4) * f32,
               gw32 = sz.gw / (p->gate_logits ? 2 : 4) * f32;
  const size_t qk32 = tokens * p->H_qk * p->d_k * f32, v32 = tokens * p->H_v * p->d_v * f32;
  const Range ins[] = {{q, sz.qk}, {k, sz.qk}, {v, sz.v}, {alpha, sz.ga}, {b, sz.gb}, {w, sz.gw},
                       {S0, sz.st}, {dO, do_bytes}, {dS_T, sz.st}};
  const Range outs[] = {{dq, qk32}, {dk, qk32}, {dv, v32}, {dalpha, ga32}, {db, gb32}, {dw, gw32}, {dS0, sz.st},
                        {workspace, ws_bytes}};
  for (int i = 0; i < 8; ++i) {
    for (const Range& r : ins)
      if (overlaps(outs[i].p, outs[i].n, r.p, r.n)) return GDN2_ERR_INVALID_ARG;
    for (int j = 0; j < i; ++j)
      if (overlaps(outs[i].p, outs[i].n, outs[j].p, outs[j].n)) return GDN2_ERR_INVALID_ARG;
  }
  const size_t need = chunk_bwd_workspace(p->B, p->H_v, p->T, p->d_k);
  if (tokens > 0 && (workspace == nullptr || ws_bytes < need)) return GDN2_ERR_WORKSPACE;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaSuccess;
  if (p->B > 0 && p->T == 0 && dS0) {
    // no token: S_T = S0, so dS0 = dS_T
    e = dS_T ? cudaMemcpyAsync(dS0, dS_T, sz.st, cudaMemcpyDeviceToDevice, s) : cudaMemsetAsync(dS0, 0, sz.st, s);
    return e == cudaSuccess ? GDN2_OK : GDN2_ERR_CUDA;
  }
  if (tokens == 0) return GDN2_OK;
  // the key-side and gate gradients are sums over CTAs (atomics)
  for (const Range& r : {Range{dq, qk32}, Range{dk, qk32}, Range{dalpha, ga32}, Range{db, gb32}})
    if (e == cudaSuccess) e = cudaMemsetAsync(const_cast<void*>(r.p), 0, r.n, s);
  if (e != cudaSuccess) return GDN2_ERR_CUDA;
  BwdArgs a;
  a.B = p->B; a.T = p->T; a.Hqk = p->H_qk; a.Hv = p->H_v;
  a.Hg = p->gate_heads == GDN2_GATE_HEADS_QK ? p->H_qk : p->H_v;
  a.gate_mode = p->gate_mode; a.gate_logits = p->gate_logits; a.scale = p->scale;
  a.q = q; a.k = k; a.v = v; a.dO = dO; a.alpha = alpha; a.b = b; a.w = w; a.S0 = S0; a.dST = dS_T;
  a.dq = dq; a.dk = dk; a.dv = dv; a.dalpha = dalpha; a.db = db; a.dw = dw; a.dS0 = dS0;
  a.ckpt = static_cast<float*>(workspace);
  e = launch_chunk_bwd(a, p->d_k, p->qkv_dtype == GDN2_BF16, p->o_dtype == GDN2_BF16, s);
  return e == cudaSuccess ? GDN2_OK : GDN2_ERR_CUDA;
}

gdn2_status gdn2_decode_step(const gdn2_params* p, const void* q, const void* k, const void* v,
                             const float* alpha, const float* b, const float* w, float* S, void* o,
                             void* stream) {
  gdn2_status st = check_common(p, true);
  if (st != GDN2_OK) return st;
  const size_t tokens = (size_t)p->B;
  if (tokens > 0) {
    if (!q || !k || !v || !o || !S) return GDN2_ERR_INVALID_ARG;
    if ((st = check_gate_ptrs(p, alpha, b, w)) != GDN2_OK) return st;
  }
  const void* ptrs[] = {q, k, v, alpha, b, w, S, o, p->conv_w};
  for (const void* ptr : ptrs)
    if (!aligned16(ptr)) return GDN2_ERR_INVALID_ARG;
  const Sizes sz = sizes(p, tokens);
  const size_t o_bytes = tokens * p->H_v * p->d_v * dsize(p->o_dtype);
  const size_t conv_bytes = ((size_t)2 * p->H_qk * p->d_k + (size_t)p->H_v * p->d_v) * 4 * sizeof(float);
  const Range ins[] = {{q, sz.qk}, {k, sz.qk}, {v, sz.v}, {alpha, sz.ga}, {b, sz.gb}, {w, sz.gw},
                       {p->conv_w, conv_bytes}};
  for (const Range& r : ins) {
    if (overlaps(o, o_bytes, r.p, r.n)) return GDN2_ERR_INVALID_ARG;
    if (overlaps(S, sz.st, r.p, r.n)) return GDN2_ERR_INVALID_ARG;
  }
  if (overlaps(o, o_bytes, S, sz.st)) return GDN2_ERR_INVALID_ARG;
  {
    const Range outs[] = {{o, o_bytes}, {S, sz.st}};
    if ((st = check_conv_state(p, ins, 7, outs, 2)) != GDN2_OK) return st;
  }
  if (tokens == 0) return GDN2_OK;

  DecodeArgs a;
  a.B = p->B; a.Hqk = p->H_qk; a.Hv = p->H_v; a.d = p->d_k; a.scale = p->scale;
  a.gate_mode = p->gate_mode; a.l2norm = p->l2norm_qk != 0; a.gate_logits = p->gate_logits;
  a.q = q; a.k = k; a.v = v; a.alpha = alpha; a.b = b; a.w = w; a.S = S; a.o = o;
  a.conv_w = p->conv_w; a.conv_in = p->conv_state_in; a.conv_out = p->conv_state_out;
  a.Hg = p->gate_heads == GDN2_GATE_HEADS_QK ? p->H_qk : p->H_v;
  cudaError_t e = launch_decode(a, p->qkv_dtype == GDN2_BF16, p->o_dtype == GDN2_BF16,
                                static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? GDN2_OK : GDN2_ERR_CUDA;
}

}  // extern "C"
