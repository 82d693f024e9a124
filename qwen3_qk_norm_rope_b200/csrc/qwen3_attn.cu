// qwen3_attn.cu - the C ABI of libqwen3attn.so: argument checks, RoPE constants, TMA
// tensor maps and kernel launches.  All device work lives in the kernels included below;
// this file does no arithmetic on tensor data.
#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include <nvtx3/nvToolsExt.h>

#include "common.cuh"
#include "decode.cuh"
#include "paged.cuh"
#include "prefill.cuh"
#include "prologue.cuh"
#include "qkv_proj.cuh"
#include "varlen.cuh"

namespace {

using q3::kD;

// A named NVTX range around each compute entry point, so a profiler's timeline shows the
// library's calls by name (header-only NVTX: nothing happens unless a tool is attached).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

constexpr int kDecodeSplit = 1024;  // keys per split-KV CTA
constexpr int kMaxDevices = 64;

uint64_t initial_wait_ns() {
  const char* e = std::getenv("QWEN3_ATTN_WAIT_NS");
  if (e != nullptr) {
    const unsigned long long v = std::strtoull(e, nullptr, 10);
    if (v > 0) return v;
  }
  return 2000000000ull;
}

uint64_t g_wait_ns = initial_wait_ns();
uint64_t g_launch_id = 0;
int g_fault = 0;
int g_softmax_path = QWEN3_SOFTMAX_AUTO;
int g_sm_pairs = QWEN3_SM_PAIRS_AUTO;
std::mutex g_mu;

q3::WaitCfg next_wait_cfg() {
  std::lock_guard<std::mutex> lk(g_mu);
  return q3::WaitCfg{g_wait_ns, ++g_launch_id};
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool is_pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }

int ilog2(int x) {
  int r = 0;
  while ((1 << r) < x) ++r;
  return r;
}

// Rotary frequencies in double (inv_i = theta^(-2i/d), or a caller's table), each split
// into a float and the float of its remainder.
q3::RopeTable make_rope_table(float theta, const double* inv_freq = nullptr) {
  q3::RopeTable t;
  for (int i = 0; i < q3::kHalf; ++i) {
    const double inv = inv_freq != nullptr ? inv_freq[i] : std::pow(static_cast<double>(theta), -2.0 * i / kD);
    t.hi[i] = static_cast<float>(inv);
    t.lo[i] = static_cast<float>(inv - static_cast<double>(t.hi[i]));
  }
  return t;
}

// A checked qwen3_attn_variant: the rotary table, the scale on cos/sin, the window.
struct Variant {
  q3::RopeTable rope;
  float scale = 1.0f;
  int window = 0;
};

int make_variant(const qwen3_attn_variant* v, Variant& out) {
  if (v == nullptr) return QWEN3_ERR_INVALID_ARG;
  if (v->inv_freq == nullptr && !(v->theta > 0.f)) return QWEN3_ERR_INVALID_ARG;
  if (!(v->attention_scaling > 0.f) || !std::isfinite(v->attention_scaling)) return QWEN3_ERR_INVALID_ARG;
  if (v->window < 0) return QWEN3_ERR_INVALID_ARG;
  if (v->inv_freq != nullptr)
    for (int i = 0; i < q3::kHalf; ++i)
      if (!std::isfinite(v->inv_freq[i]) || std::fabs(v->inv_freq[i]) >= 1e30) return QWEN3_ERR_INVALID_ARG;
  out.rope = make_rope_table(v->theta, v->inv_freq);
  out.scale = v->attention_scaling;
  out.window = v->window;
  return QWEN3_OK;
}

// A checked qwen3_paged_kv.
struct PagedKV {
  qwen3_bf16* k = nullptr;
  qwen3_bf16* v = nullptr;
  const int32_t* table = nullptr;
  int num_pages = 0, page = 0, max_blocks = 0, log2_page = 0;
};

int make_paged(const qwen3_paged_kv* kv, int Hkv, PagedKV& out) {
  if (kv == nullptr || kv->k_pages == nullptr || kv->v_pages == nullptr || kv->block_table == nullptr)
    return QWEN3_ERR_INVALID_ARG;
  if (kv->num_pages <= 0 || kv->max_blocks <= 0 || kv->page_size < 16 || kv->page_size > 1024 ||
      (kv->page_size & (kv->page_size - 1)) != 0)
    return QWEN3_ERR_INVALID_ARG;
  if (!aligned(kv->k_pages, 16) || !aligned(kv->v_pages, 16) || !aligned(kv->block_table, 4))
    return QWEN3_ERR_INVALID_ARG;
  // rows of d in a pool must index as int32 (TMA row coordinates)
  if (static_cast<long long>(kv->num_pages) * Hkv * kv->page_size > 0x7fffffffLL) return QWEN3_ERR_UNSUPPORTED;
  if (static_cast<long long>(kv->max_blocks) * kv->page_size > 0x7fffffffLL) return QWEN3_ERR_UNSUPPORTED;
  out.k = kv->k_pages;
  out.v = kv->v_pages;
  out.table = kv->block_table;
  out.num_pages = kv->num_pages;
  out.page = kv->page_size;
  out.max_blocks = kv->max_blocks;
  out.log2_page = ilog2(kv->page_size);
  return QWEN3_OK;
}

// The default rope type with base theta, full causal attention.
int theta_variant(float theta, Variant& out) {
  qwen3_attn_variant v;
  v.theta = theta;
  v.inv_freq = nullptr;
  v.attention_scaling = 1.0f;
  v.window = 0;
  return make_variant(&v, out);
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// bf16 tiled map, 128B swizzle, zero fill out of bounds.  dims/strides innermost first;
// strides[i] is the byte stride of dim i+1.
bool make_map(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims, const cuuint64_t* strides,
              const cuuint32_t* box) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, static_cast<cuuint32_t>(rank), const_cast<void*>(base), dims,
            strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Opt the big-shared-memory kernels in once per device.
int ensure_kernel_attrs() {
  static bool done[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return QWEN3_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  if (done[dev]) return QWEN3_OK;
  if (cudaFuncSetAttribute(q3::fmha_prefill_kernel<false, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           q3::kPrefillSmemBytes) != cudaSuccess ||
      cudaFuncSetAttribute(q3::fmha_prefill_kernel<true, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           q3::kPrefillSmemBytes) != cudaSuccess ||
      cudaFuncSetAttribute(q3::fmha_prefill_kernel<false, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           q3::kPrefillSmemBytes) != cudaSuccess ||
      cudaFuncSetAttribute(q3::fmha_prefill_kernel<true, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           q3::kPrefillSmemBytes) != cudaSuccess ||
      cudaFuncSetAttribute(q3::fmha_prefill_kernel<false, false, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           q3::kPrefillSmemBytes) != cudaSuccess)
    return QWEN3_ERR_CUDA;
  if (cudaFuncSetAttribute(q3::decode_split_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           q3::kDecodeSmemBytes) != cudaSuccess ||
      cudaFuncSetAttribute(q3::decode_split_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           q3::kDecodeSmemBytes) != cudaSuccess)
    return QWEN3_ERR_CUDA;
  if (cudaFuncSetAttribute(q3::qkv_proj_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           q3::kQkvSmemBytes) != cudaSuccess ||
      cudaFuncSetAttribute(q3::qkv_proj_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           q3::kQkv2SmemBytes) != cudaSuccess)
    return QWEN3_ERR_CUDA;
  done[dev] = true;
  return QWEN3_OK;
}

// Streaming multiprocessors of the current device (148 on B200), cached per device.
int num_sms() {
  static int sms[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
  if (sms[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    sms[dev] = n;
  }
  return sms[dev];
}

// Bytes of the K' region of the prefill workspace (rounded to keep what follows aligned).
size_t kspace_bytes(int B, int T, int Hkv, int d) {
  return (static_cast<size_t>(B) * Hkv * T * d * 2 + 255) & ~static_cast<size_t>(255);
}

// Key-axis split of a prefill whose work items are few next to the SMs (a short chunk over
// a long cached prefix): the number of runs its keys are cut into, 1 for no split.  It is
// fixed by the shapes alone, so the workspace size that holds the partials is known on the
// host: about kSplitTarget items in all, each run at least 4 key tiles, at most 32 runs.
// When every (batch row, KV head) has a single query tile (T <= 128 / G, single_qtile), the
// kernel's K/V ring takes a third stage, and with kDualRuns an item takes two runs, one per
// softmax group, so the count is even and twice the items'.
constexpr int kSplitTarget = 128;
constexpr bool kDualRuns = true;
bool single_qtile(int T, int Hq, int Hkv) { return static_cast<long long>(T) * (Hq / Hkv) <= 128; }
bool dual_split(int T, int Hq, int Hkv) { return kDualRuns && single_qtile(T, Hq, Hkv); }
int split_count(int B, int start, int T, int Hq, int Hkv, int window) {
  if (window > 0 || B <= 0 || T <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0) return 1;
  const int G = Hq / Hkv;
  if (G > 128) return 1;
  const long long P = 128 / G;
  const long long n_pairs = ((T + P - 1) / P + 1) / 2;
  const long long items = static_cast<long long>(B) * Hkv * n_pairs;
  const long long tiles = (static_cast<long long>(start) + T + 127) / 128;
  if (tiles < 8) return 1;
  if (dual_split(T, Hq, Hkv)) {
    if (items > kSplitTarget) return 1;
    long long n = std::min<long long>(2 * kSplitTarget / items, tiles / 4);
    n = std::min<long long>(n, 32) & ~1LL;
    return n >= 2 ? static_cast<int>(n) : 1;
  }
  if (items * 2 > kSplitTarget) return 1;
  long long n = std::min<long long>(kSplitTarget / items, tiles / 4);
  n = std::min<long long>(n, 32);
  return n >= 2 ? static_cast<int>(n) : 1;
}

// Bytes of the split partials: O/l fp32 [B*T, Hq, n, d] and LSEs [B*T, Hq, n], each
// 256-byte aligned.
size_t split_bytes(int B, int T, int Hq, int n) {
  if (n <= 1) return 0;
  const size_t rows = static_cast<size_t>(B) * T * Hq * n;
  return ((rows * kD * 4 + 255) & ~static_cast<size_t>(255)) + ((rows * 4 + 255) & ~static_cast<size_t>(255));
}

// Pages of at least this many keys are read in place by the prefill attention kernel (one
// TMA box per page per 64-dim half); smaller ones are gathered first, since a tile of them
// would take too many small boxes.
constexpr int kInPlaceMinPage = 64;

int check_common(int Hq, int Hkv, int d) {
  if (Hq <= 0 || Hkv <= 0) return QWEN3_ERR_INVALID_ARG;
  if (d != kD) return QWEN3_ERR_UNSUPPORTED;
  if (Hq % Hkv != 0 || !is_pow2(Hq / Hkv)) return QWEN3_ERR_UNSUPPORTED;
  return QWEN3_OK;
}

// Q (optional, the prefill): raw xq [B, T, Hq, d] with gain wq to Q' [B, H, T*Hq/H, d].
struct PrologueQ {
  const void* xq = nullptr;
  const float* wq = nullptr;
  void* dstq = nullptr;
  int Hq = 0;
};

// A varlen batch (optional): token offsets [B + 1] and, with pages, the checked metadata.
struct PrologueVarlen {
  const int32_t* cu = nullptr;
  const int4* seq = nullptr;
  int B = 0;
};

int launch_prologue(const void* x, const float* w, const int32_t* pos, void* dst, const void* v_src, void* v_dst,
                    int B, int T, int H, int Tcap, int write_at_pos, const Variant& var, float eps,
                    cudaStream_t stream, const PrologueQ& q = PrologueQ(), const PagedKV* pg = nullptr,
                    int key0 = 0, const PrologueVarlen& vl = PrologueVarlen()) {
  q3::PrologueParams p;
  p.x = static_cast<const uint32_t*>(x);
  p.w = w;
  p.pos = pos;
  p.dst = static_cast<uint32_t*>(dst);
  p.v_src = static_cast<const uint2*>(v_src);
  p.v_dst = static_cast<uint2*>(v_dst);
  p.xq = static_cast<const uint32_t*>(q.xq);
  p.wq = q.wq;
  p.dstq = static_cast<uint32_t*>(q.dstq);
  p.Hq = q.Hq;
  p.log2G = q.xq != nullptr ? ilog2(q.Hq / H) : 0;
  p.B = B;
  p.T = T;
  p.H = H;
  p.Tcap = Tcap;
  p.write_at_pos = write_at_pos;
  p.eps = eps;
  p.rope_scale = var.scale;
  p.rope = var.rope;
  p.block_table = pg != nullptr ? pg->table : nullptr;
  p.max_blocks = pg != nullptr ? pg->max_blocks : 0;
  p.log2_page = pg != nullptr ? pg->log2_page : 0;
  p.num_pages = pg != nullptr ? pg->num_pages : 0;
  p.key0 = key0;
  p.vl_cu = vl.cu;
  p.vl_seq = vl.seq;
  p.vl_B = vl.B;
  const long long ntok = static_cast<long long>(B) * T;
  if (ntok > 0x7fffffffLL) return QWEN3_ERR_UNSUPPORTED;
  const int warps = 8;
  // A warp per token, or per batch of a token's heads when that still fits one wave of
  // resident warps (32 per SM): few tokens then run their batches side by side.
  const long long nb = (H + q3::kPrologueHeads - 1) / q3::kPrologueHeads +
                       (q.xq != nullptr ? (q.Hq + q3::kPrologueHeads - 1) / q3::kPrologueHeads : 0);
  const bool per_batch = nb > 1 && ntok * nb <= static_cast<long long>(num_sms()) * 32;
  const long long units = per_batch ? ntok * nb : ntok;
  long long blocks = (units + warps - 1) / warps;
  const long long cap = static_cast<long long>(num_sms()) * 16;  // grid-stride beyond 16 blocks per SM
  if (blocks > cap) blocks = cap;
  if (per_batch)
    q3::qk_norm_rope_kernel<true><<<static_cast<unsigned>(blocks), warps * 32, 0, stream>>>(p);
  else
    q3::qk_norm_rope_kernel<false><<<static_cast<unsigned>(blocks), warps * 32, 0, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? QWEN3_OK : QWEN3_ERR_CUDA;
}

}  // namespace

extern "C" {

const char* qwen3_attn_version(void) { return "qwen3-attn-b200 0.1 (sm_100a)"; }

const char* qwen3_attn_status_string(int status) {
  switch (status) {
    case QWEN3_OK: return "ok";
    case QWEN3_ERR_INVALID_ARG: return "invalid argument";
    case QWEN3_ERR_UNSUPPORTED: return "unsupported shape";
    case QWEN3_ERR_CUDA: return "CUDA runtime or launch failure";
    case QWEN3_ERR_DEVICE_TIMEOUT: return "bounded device-side wait ran out";
    case QWEN3_ERR_WORKSPACE: return "workspace missing or too small";
    default: return "unknown status";
  }
}

uint64_t qwen3_attn_set_wait_limit(uint64_t ns) {
  std::lock_guard<std::mutex> lk(g_mu);
  const uint64_t old = g_wait_ns;
  g_wait_ns = ns;
  return old;
}

void qwen3_attn_set_fault_injection(int flags) {
  std::lock_guard<std::mutex> lk(g_mu);
  g_fault = flags;
}

int qwen3_attn_set_softmax_path(int path) {
  if (path != QWEN3_SOFTMAX_AUTO && path != QWEN3_SOFTMAX_RUNNING_MAX) return -1;
  std::lock_guard<std::mutex> lk(g_mu);
  const int old = g_softmax_path;
  g_softmax_path = path;
  return old;
}

int qwen3_attn_set_sm_pairs(int mode) {
  if (mode != QWEN3_SM_PAIRS_AUTO && mode != QWEN3_SM_PAIRS_OFF && mode != QWEN3_SM_PAIRS_ALWAYS) return -1;
  std::lock_guard<std::mutex> lk(g_mu);
  const int old = g_sm_pairs;
  g_sm_pairs = mode;
  return old;
}

int qwen3_attn_device_status(qwen3_stream_t stream, int clear, int* site) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return QWEN3_ERR_CUDA;
  int h[2] = {0, 0};
  if (cudaMemcpyFromSymbol(h, q3::g_status, sizeof(h)) != cudaSuccess) return QWEN3_ERR_CUDA;
  if (clear) {
    const int z[2] = {0, 0};
    if (cudaMemcpyToSymbol(q3::g_status, z, sizeof(z)) != cudaSuccess) return QWEN3_ERR_CUDA;
  }
  if (site != nullptr) *site = h[1];
  return h[0];
}

size_t qwen3_attn_prefill_workspace_size(int B, int T, int Hq, int Hkv, int d) {
  if (B <= 0 || T <= 0 || Hq <= 0 || Hkv <= 0 || d <= 0) return 0;
  // K' [B, Hkv, T, d] bf16, then Q' [B, Hkv, T*G, d] bf16 (as many elements as q)
  return kspace_bytes(B, T, Hkv, d) + kspace_bytes(B, T, Hq, d) + 256;
}

size_t qwen3_attn_prefill_paged_workspace_size(int B, int start, int T, int Hq, int Hkv, int d) {
  if (B <= 0 || start < 0 || T <= 0 || Hq <= 0 || Hkv <= 0 || d <= 0) return 0;
  // K and V of the row's first start + T keys gathered out of pages under kInPlaceMinPage
  // keys (pages of that size or more are read in place and leave this region unused), Q',
  // then the partials of a key-axis split
  return 2 * kspace_bytes(B, start + T, Hkv, d) + kspace_bytes(B, T, Hq, d) +
         split_bytes(B, T, Hq, split_count(B, start, T, Hq, Hkv, 0)) + 256;
}

size_t qwen3_attn_prefill_chunk_workspace_size(int B, int start, int T, int Hq, int Hkv, int d) {
  if (B <= 0 || start < 0 || T <= 0 || Hq <= 0 || Hkv <= 0 || d <= 0) return 0;
  return qwen3_attn_prefill_workspace_size(B, T, Hq, Hkv, d) + split_bytes(B, T, Hq, split_count(B, start, T, Hq, Hkv, 0));
}

size_t qwen3_attn_decode_workspace_size(int N, int Hq, int d, int Lmax) {
  if (N <= 0 || Hq <= 0 || d <= 0 || Lmax <= 0) return 0;
  const size_t ns = (static_cast<size_t>(Lmax) + kDecodeSplit - 1) / kDecodeSplit;
  const size_t o_bytes = static_cast<size_t>(N) * Hq * ns * d * 4;
  return o_bytes + 256 + static_cast<size_t>(N) * Hq * ns * 4 + 256;
}

size_t qwen3_attn_kv_cache_bytes(int N, int Hkv, int Lmax, int d) {
  if (N <= 0 || Hkv <= 0 || Lmax <= 0 || d <= 0) return 0;
  return static_cast<size_t>(2) * N * Hkv * Lmax * d * sizeof(qwen3_bf16);
}

int qwen3_qk_norm_rope_variant(const qwen3_bf16* x, const float* w, const int32_t* pos, qwen3_bf16* dst,
                               const qwen3_bf16* v_src, qwen3_bf16* v_dst, int B, int T, int H, int d, int Tcap,
                               int write_at_pos, const qwen3_attn_variant* variant, float eps,
                               qwen3_stream_t stream) {
  NvtxRange nvtx_range("qwen3_qk_norm_rope_variant");
  Variant var;
  const int sv = make_variant(variant, var);
  if (sv != QWEN3_OK) return sv;
  if (x == nullptr || w == nullptr || pos == nullptr || dst == nullptr) return QWEN3_ERR_INVALID_ARG;
  if ((v_src == nullptr) != (v_dst == nullptr)) return QWEN3_ERR_INVALID_ARG;
  if (B <= 0 || T <= 0 || H <= 0 || Tcap <= 0) return QWEN3_ERR_INVALID_ARG;
  if (d != kD) return QWEN3_ERR_UNSUPPORTED;
  if (!write_at_pos && Tcap < T) return QWEN3_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(dst, 16) || !aligned(w, 8) || !aligned(pos, 4)) return QWEN3_ERR_INVALID_ARG;
  if (v_src != nullptr && (!aligned(v_src, 16) || !aligned(v_dst, 16))) return QWEN3_ERR_INVALID_ARG;
  if (!(eps >= 0.f)) return QWEN3_ERR_INVALID_ARG;
  return launch_prologue(x, w, pos, dst, v_src, v_dst, B, T, H, Tcap, write_at_pos, var, eps,
                         reinterpret_cast<cudaStream_t>(stream));
}

int qwen3_qk_norm_rope(const qwen3_bf16* x, const float* w, const int32_t* pos, qwen3_bf16* dst,
                       const qwen3_bf16* v_src, qwen3_bf16* v_dst, int B, int T, int H, int d, int Tcap,
                       int write_at_pos, float theta, float eps, qwen3_stream_t stream) {
  NvtxRange nvtx_range("qwen3_qk_norm_rope");
  const qwen3_attn_variant v = {theta, nullptr, 1.0f, 0};
  return qwen3_qk_norm_rope_variant(x, w, pos, dst, v_src, v_dst, B, T, H, d, Tcap, write_at_pos, &v, eps, stream);
}

namespace {

// Prefill of T new tokens per batch row after `start` cached ones (start > 0 needs the caches).
// With `pg`, the cache is paged: the new keys and values go into the pages, and the attention
// kernel reads the row's start + T keys and values there, page by page.
// The attention kernel, persistent (one CTA per SM, fewer for fewer items), as a
// programmatic dependent launch: its CTAs may be scheduled while the kernel before it
// finishes; they set up (barriers, TMEM, tensor maps, the logit bound) and wait
// (griddepcontrol.wait) before their first load of Q', K' or the cache.
int launch_fmha(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& mo,
                const q3::PrefillParams& p, int max_items, bool window, bool varlen, cudaStream_t s,
                bool split = false) {
  const int grid = max_items < num_sms() ? max_items : num_sms();
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(q3::kPrefillThreads);
  cfg.dynamicSmemBytes = q3::kPrefillSmemBytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t le;
  if (split)
    le = cudaLaunchKernelEx(&cfg, q3::fmha_prefill_kernel<false, false, true>, mq, mk, mv, mo, p);
  else if (varlen)
    le = window ? cudaLaunchKernelEx(&cfg, q3::fmha_prefill_kernel<true, true>, mq, mk, mv, mo, p)
                : cudaLaunchKernelEx(&cfg, q3::fmha_prefill_kernel<false, true>, mq, mk, mv, mo, p);
  else
    le = window ? cudaLaunchKernelEx(&cfg, q3::fmha_prefill_kernel<true, false>, mq, mk, mv, mo, p)
                : cudaLaunchKernelEx(&cfg, q3::fmha_prefill_kernel<false, false>, mq, mk, mv, mo, p);
  if (le != cudaSuccess) {
    (void)cudaGetLastError();
    return QWEN3_ERR_CUDA;
  }
  return cudaGetLastError() == cudaSuccess ? QWEN3_OK : QWEN3_ERR_CUDA;
}

int prefill_impl(const qwen3_bf16* q, const qwen3_bf16* k, const qwen3_bf16* v, const float* q_norm_w,
                 const float* k_norm_w, const int32_t* pos, qwen3_bf16* out, float* lse, qwen3_bf16* k_cache,
                 qwen3_bf16* v_cache, int start, int Tcap, void* workspace, size_t ws_bytes, int B, int T, int Hq,
                 int Hkv, int d, const Variant& var, float eps, qwen3_stream_t stream,
                 const PagedKV* pg = nullptr) {
  if (q == nullptr || k == nullptr || v == nullptr || q_norm_w == nullptr || k_norm_w == nullptr ||
      pos == nullptr || out == nullptr)
    return QWEN3_ERR_INVALID_ARG;
  if (B <= 0 || T <= 0) return QWEN3_ERR_INVALID_ARG;
  int st = check_common(Hq, Hkv, d);
  if (st != QWEN3_OK) return st;
  if (Hq / Hkv > 128) return QWEN3_ERR_UNSUPPORTED;
  if ((k_cache == nullptr) != (v_cache == nullptr)) return QWEN3_ERR_INVALID_ARG;
  if (pg != nullptr && k_cache != nullptr) return QWEN3_ERR_INVALID_ARG;
  const bool use_cache = k_cache != nullptr;
  if (start < 0 || (start > 0 && !use_cache && pg == nullptr)) return QWEN3_ERR_INVALID_ARG;
  if (use_cache && (Tcap <= 0 || static_cast<long long>(start) + T > Tcap)) return QWEN3_ERR_INVALID_ARG;
  if (pg != nullptr && static_cast<long long>(start) + T > static_cast<long long>(pg->max_blocks) * pg->page)
    return QWEN3_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) || !aligned(q_norm_w, 8) ||
      !aligned(k_norm_w, 8) || !aligned(pos, 4) || (lse != nullptr && !aligned(lse, 4)))
    return QWEN3_ERR_INVALID_ARG;
  if (use_cache && (!aligned(k_cache, 16) || !aligned(v_cache, 16))) return QWEN3_ERR_INVALID_ARG;
  if (!(eps >= 0.f)) return QWEN3_ERR_INVALID_ARG;
  // A key-axis split when the work items are few; its partials follow the other regions
  // of the workspace, and a workspace without room for them runs the call unsplit.
  int n_split = split_count(B, start, T, Hq, Hkv, var.window);
  const bool in_place = pg != nullptr && pg->page >= kInPlaceMinPage;
  const size_t base = pg == nullptr ? qwen3_attn_prefill_workspace_size(B, T, Hq, Hkv, d)
                      : in_place    ? kspace_bytes(B, T, Hq, d) + 256  // Q' only: K, V are read in place
                                    : 2 * kspace_bytes(B, start + T, Hkv, d) + kspace_bytes(B, T, Hq, d) + 256;
  if (workspace == nullptr || base == 0 || ws_bytes < base) return QWEN3_ERR_WORKSPACE;
  if (ws_bytes < base + split_bytes(B, T, Hq, n_split)) n_split = 1;
  if (static_cast<long long>(T) * Hq > (1LL << 31) / kD || static_cast<long long>(B) * Hkv > 65535LL * 1024)
    return QWEN3_ERR_UNSUPPORTED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if ((st = ensure_kernel_attrs()) != QWEN3_OK) return st;

  // 1. QK prologue.  K' in cache layout [B, Hkv, Tc, d] from slot `start` on (and V copied
  //    when filling a cache; shifting the base by start rows puts token t at slot start + t),
  //    and Q' in the query tiles' row order [B, Hkv, T*G, d], both in one pass per token.
  const uintptr_t w0 = (reinterpret_cast<uintptr_t>(workspace) + 255) & ~static_cast<uintptr_t>(255);
  qwen3_bf16* kdst = use_cache ? k_cache : reinterpret_cast<qwen3_bf16*>(w0);
  qwen3_bf16* vsrc = use_cache ? v_cache : nullptr;  // V in cache layout, when not read raw
  qwen3_bf16* qdst = reinterpret_cast<qwen3_bf16*>(w0 + kspace_bytes(B, T, Hkv, d));
  int Tc = use_cache ? Tcap : T;
  const size_t shift = static_cast<size_t>(start) * kD;
  PrologueQ pq;
  pq.xq = q;
  pq.wq = q_norm_w;
  pq.dstq = qdst;
  pq.Hq = Hq;
  if (pg == nullptr) {
    st = launch_prologue(k, k_norm_w, pos, kdst + shift, use_cache ? v : nullptr,
                         use_cache ? v_cache + shift : nullptr, B, T, Hkv, Tc, 0, var, eps, s, pq);
    if (st != QWEN3_OK) return st;
  } else {
    // Paged: K' and V of the new tokens into their pages (keys start..start+T-1), Q' into the
    // workspace.  The attention kernel then reads the row's start + T keys and values in
    // place, page by page; pages under kInPlaceMinPage keys are first gathered into the
    // workspace, [B, Hkv, start + T, d] each, where the attention reads them.
    const int n = start + T;
    qdst = reinterpret_cast<qwen3_bf16*>(in_place ? w0 : w0 + 2 * kspace_bytes(B, n, Hkv, d));
    pq.dstq = qdst;
    st = launch_prologue(k, k_norm_w, pos, pg->k, v, pg->v, B, T, Hkv, 1, 0, var, eps, s, pq, pg, start);
    if (st != QWEN3_OK) return st;
    if (!in_place) {
      if (static_cast<long long>(B) * Hkv * n > (1LL << 31) / kD) return QWEN3_ERR_UNSUPPORTED;
      kdst = reinterpret_cast<qwen3_bf16*>(w0);
      vsrc = reinterpret_cast<qwen3_bf16*>(w0 + kspace_bytes(B, n, Hkv, d));
      Tc = n;
      q3::GatherParams gp;
      gp.k_pages = reinterpret_cast<const uint4*>(pg->k);
      gp.v_pages = reinterpret_cast<const uint4*>(pg->v);
      gp.block_table = pg->table;
      gp.k_out = reinterpret_cast<uint4*>(kdst);
      gp.v_out = reinterpret_cast<uint4*>(vsrc);
      gp.B = B;
      gp.Hkv = Hkv;
      gp.n = n;
      gp.max_blocks = pg->max_blocks;
      gp.log2_page = pg->log2_page;
      gp.num_pages = pg->num_pages;
      const long long chunks = static_cast<long long>(B) * n * Hkv * 16;
      long long blocks = (chunks + 255) / 256;
      if (blocks > static_cast<long long>(num_sms()) * 32) blocks = static_cast<long long>(num_sms()) * 32;
      q3::paged_gather_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(gp);
      if (cudaGetLastError() != cudaSuccess) return QWEN3_ERR_CUDA;
    }
  }

  // 2. Tensor maps.  The key-axis extent is start + T (not Tcap) so slots past the new tokens
  //    read as zeros.
  CUtensorMap mq, mk, mv, mo;
  const cuuint32_t box[4] = {64, 128, 1, 1};
  {
    // out [B, T, Hq, d] as boxes of [P positions][G heads][64 dims]: one query tile's half
    const int G = Hq / Hkv;
    const cuuint64_t odims[4] = {static_cast<cuuint64_t>(kD), static_cast<cuuint64_t>(Hq),
                                 static_cast<cuuint64_t>(T), static_cast<cuuint64_t>(B)};
    const cuuint64_t ostr[3] = {kD * 2ull, static_cast<cuuint64_t>(Hq) * kD * 2ull,
                                static_cast<cuuint64_t>(T) * Hq * kD * 2ull};
    const cuuint32_t obox[4] = {64, static_cast<cuuint32_t>(G), static_cast<cuuint32_t>(128 / G), 1};
    if (!make_map(&mo, out, 4, odims, ostr, obox)) return QWEN3_ERR_CUDA;
  }
  {
    // Q' rows past T*G read as zeros (their outputs are never stored)
    const cuuint64_t TG = static_cast<cuuint64_t>(T) * (Hq / Hkv);
    const cuuint64_t qdims[4] = {static_cast<cuuint64_t>(kD), TG, static_cast<cuuint64_t>(Hkv),
                                 static_cast<cuuint64_t>(B)};
    const cuuint64_t qstr[3] = {kD * 2ull, TG * kD * 2ull, static_cast<cuuint64_t>(Hkv) * TG * kD * 2ull};
    if (!make_map(&mq, qdst, 4, qdims, qstr, box)) return QWEN3_ERR_CUDA;
  }
  if (in_place) {
    // the page pools as rows of d, boxes of one page (or 128 rows of a larger page)
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(kD),
                                static_cast<cuuint64_t>(pg->num_pages) * Hkv * pg->page};
    const cuuint64_t str[1] = {kD * 2ull};
    const cuuint32_t pbox[2] = {64, static_cast<cuuint32_t>(std::min(pg->page, 128))};
    if (!make_map(&mk, pg->k, 2, dims, str, pbox) || !make_map(&mv, pg->v, 2, dims, str, pbox))
      return QWEN3_ERR_CUDA;
  } else {
    const cuuint64_t dims[4] = {static_cast<cuuint64_t>(kD), static_cast<cuuint64_t>(start) + T,
                                static_cast<cuuint64_t>(Hkv), static_cast<cuuint64_t>(B)};
    const cuuint64_t str[3] = {kD * 2ull, static_cast<cuuint64_t>(Tc) * kD * 2ull,
                               static_cast<cuuint64_t>(Hkv) * Tc * kD * 2ull};
    if (!make_map(&mk, kdst, 4, dims, str, box)) return QWEN3_ERR_CUDA;
    if (vsrc != nullptr) {
      if (!make_map(&mv, vsrc, 4, dims, str, box)) return QWEN3_ERR_CUDA;
    } else {
      const cuuint64_t vstr[3] = {static_cast<cuuint64_t>(Hkv) * kD * 2ull, kD * 2ull,
                                  static_cast<cuuint64_t>(T) * Hkv * kD * 2ull};
      if (!make_map(&mv, v, 4, dims, vstr, box)) return QWEN3_ERR_CUDA;
    }
  }

  // 3. Attention.
  q3::PrefillParams p{};
  p.q_norm_w = q_norm_w;
  p.k_norm_w = k_norm_w;
  p.lse = lse;
  p.B = B;
  p.T = T;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.log2G = ilog2(Hq / Hkv);
  p.P = 128 >> p.log2G;
  p.n_qt = (T + p.P - 1) / p.P;
  p.n_pairs = (p.n_qt + 1) / 2;
  const long long n_items = static_cast<long long>(p.n_pairs) * B * Hkv;
  if (n_items > 0x7fffffffLL) return QWEN3_ERR_UNSUPPORTED;
  p.n_items = static_cast<int>(n_items);
  p.start = start;
  p.window = var.window;
  p.rope_scale = var.scale;
  p.eps = eps;
  p.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(kD)));
  p.wait = next_wait_cfg();
  {
    std::lock_guard<std::mutex> lk(g_mu);
    p.fault = g_fault;
    p.force_rmax = g_softmax_path == QWEN3_SOFTMAX_RUNNING_MAX ? 1 : 0;
  }
  if (in_place) {
    p.block_table = pg->table;
    p.max_blocks = pg->max_blocks;
    p.log2_page = pg->log2_page;
    p.num_pages = pg->num_pages;
  }
  // A contiguous cache's keys and values before `start` come from earlier calls; a gathered
  // copy of pages is written by this call's gather kernel.
  p.kv_early = (pg == nullptr && use_cache) ? 1 : 0;
  p.n_split = n_split;
  if (n_split <= 1) return launch_fmha(mq, mk, mv, mo, p, static_cast<int>(n_items), var.window > 0, false, s);

  // 4. Key-axis split: every item leaves partials, which one more kernel merges.
  const uintptr_t pbase = (w0 + base - 256 + 255) & ~static_cast<uintptr_t>(255);
  const size_t rows = static_cast<size_t>(B) * T * Hq * n_split;
  p.part_o = reinterpret_cast<float*>(pbase);
  p.part_lse = reinterpret_cast<float*>(pbase + ((rows * kD * 4 + 255) & ~static_cast<size_t>(255)));
  p.dual = dual_split(T, Hq, Hkv) ? 1 : 0;  // n_split is even then
  p.ring3 = single_qtile(T, Hq, Hkv) ? 1 : 0;
  const long long split_items = n_items * (p.dual ? n_split / 2 : n_split);
  if (split_items > 0x7fffffffLL) return QWEN3_ERR_UNSUPPORTED;
  p.n_items = static_cast<int>(split_items);
  if ((st = launch_fmha(mq, mk, mv, mo, p, static_cast<int>(split_items), false, false, s, true)) != QWEN3_OK)
    return st;
  q3::SplitCombineParams c;
  c.part_o = p.part_o;
  c.part_lse = p.part_lse;
  c.out = reinterpret_cast<uint2*>(out);
  c.lse = lse;
  c.B = B;
  c.T = T;
  c.Hq = Hq;
  c.n_split = n_split;
  const long long nrow = static_cast<long long>(B) * T * Hq;
  cudaLaunchConfig_t cfg = {};
  if (nrow > 0x7fffffffLL) return QWEN3_ERR_UNSUPPORTED;
  cfg.gridDim = dim3(static_cast<unsigned>(nrow));  // a block per (token, head)
  cfg.blockDim = dim3(q3::kCombineWarps * 32);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, q3::prefill_split_combine_kernel, c) != cudaSuccess) {
    (void)cudaGetLastError();
    return QWEN3_ERR_CUDA;
  }
  return cudaGetLastError() == cudaSuccess ? QWEN3_OK : QWEN3_ERR_CUDA;
}

}  // namespace

int qwen3_attn_prefill_ex(const qwen3_bf16* q, const qwen3_bf16* k, const qwen3_bf16* v, const float* q_norm_w,
                          const float* k_norm_w, const int32_t* pos, qwen3_bf16* out, float* lse,
                          qwen3_bf16* k_cache, qwen3_bf16* v_cache, int Tcap, void* workspace, size_t ws_bytes,
                          int B, int T, int Hq, int Hkv, int d, float theta, float eps, qwen3_stream_t stream) {
  NvtxRange nvtx_range("qwen3_attn_prefill_ex");
  Variant var;
  const int sv = theta_variant(theta, var);
  if (sv != QWEN3_OK) return sv;
  return prefill_impl(q, k, v, q_norm_w, k_norm_w, pos, out, lse, k_cache, v_cache, 0, Tcap, workspace, ws_bytes,
                      B, T, Hq, Hkv, d, var, eps, stream);
}

int qwen3_attn_prefill_variant(const qwen3_bf16* q, const qwen3_bf16* k, const qwen3_bf16* v, const float* q_norm_w,
                               const float* k_norm_w, const int32_t* pos, qwen3_bf16* out, float* lse,
                               qwen3_bf16* k_cache, qwen3_bf16* v_cache, int start, int Tcap, void* workspace,
                               size_t ws_bytes, int B, int T, int Hq, int Hkv, int d,
                               const qwen3_attn_variant* variant, float eps, qwen3_stream_t stream) {
  NvtxRange nvtx_range("qwen3_attn_prefill_variant");
  Variant var;
  const int sv = make_variant(variant, var);
  if (sv != QWEN3_OK) return sv;
  return prefill_impl(q, k, v, q_norm_w, k_norm_w, pos, out, lse, k_cache, v_cache, start, Tcap, workspace,
                      ws_bytes, B, T, Hq, Hkv, d, var, eps, stream);
}

int qwen3_attn_prefill_chunk(const qwen3_bf16* q, const qwen3_bf16* k, const qwen3_bf16* v, const float* q_norm_w,
                             const float* k_norm_w, const int32_t* pos, qwen3_bf16* out, float* lse,
                             qwen3_bf16* k_cache, qwen3_bf16* v_cache, int start, int Tcap, void* workspace,
                             size_t ws_bytes, int B, int T, int Hq, int Hkv, int d, float theta, float eps,
                             qwen3_stream_t stream) {
  NvtxRange nvtx_range("qwen3_attn_prefill_chunk");
  if (k_cache == nullptr || v_cache == nullptr) return QWEN3_ERR_INVALID_ARG;
  Variant var;
  const int sv = theta_variant(theta, var);
  if (sv != QWEN3_OK) return sv;
  return prefill_impl(q, k, v, q_norm_w, k_norm_w, pos, out, lse, k_cache, v_cache, start, Tcap, workspace,
                      ws_bytes, B, T, Hq, Hkv, d, var, eps, stream);
}

int qwen3_attn_prefill(const qwen3_bf16* q, const qwen3_bf16* k, const qwen3_bf16* v, const float* q_norm_w,
                       const float* k_norm_w, const int32_t* pos, qwen3_bf16* out, int B, int T, int Hq, int Hkv,
                       int d, float theta, float eps, qwen3_stream_t stream) {
  NvtxRange nvtx_range("qwen3_attn_prefill");
  if (q == nullptr || k == nullptr || v == nullptr || q_norm_w == nullptr || k_norm_w == nullptr ||
      pos == nullptr || out == nullptr || B <= 0 || T <= 0)
    return QWEN3_ERR_INVALID_ARG;
  const int st0 = check_common(Hq, Hkv, d);
  if (st0 != QWEN3_OK) return st0;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const size_t bytes = qwen3_attn_prefill_workspace_size(B, T, Hq, Hkv, d);
  void* ws = nullptr;
  if (cudaMallocAsync(&ws, bytes, s) != cudaSuccess) return QWEN3_ERR_CUDA;
  const int st = qwen3_attn_prefill_ex(q, k, v, q_norm_w, k_norm_w, pos, out, nullptr, nullptr, nullptr, 0, ws,
                                       bytes, B, T, Hq, Hkv, d, theta, eps, stream);
  const bool freed = cudaFreeAsync(ws, s) == cudaSuccess;
  if (st != QWEN3_OK) return st;
  return freed ? QWEN3_OK : QWEN3_ERR_CUDA;
}

}  // extern "C"

namespace {

// The host checks of a decode call's tensors and sizes (every one but the workspace's).
int decode_check(const qwen3_bf16* q, const qwen3_bf16* k_new, const qwen3_bf16* v_new, const float* q_norm_w,
                 const float* k_norm_w, const qwen3_bf16* k_cache, const qwen3_bf16* v_cache,
                 const int32_t* cache_lens, const qwen3_bf16* out, const float* lse, int N, int Hq, int Hkv, int d,
                 int Lmax, float eps, bool paged) {
  if (q == nullptr || k_new == nullptr || v_new == nullptr || q_norm_w == nullptr || k_norm_w == nullptr ||
      k_cache == nullptr || v_cache == nullptr || cache_lens == nullptr || out == nullptr)
    return QWEN3_ERR_INVALID_ARG;
  if (N <= 0 || Lmax <= 0) return QWEN3_ERR_INVALID_ARG;
  const int st = check_common(Hq, Hkv, d);
  if (st != QWEN3_OK) return st;
  if (Hq / Hkv > 16 || N > 65535 || Hkv > 65535) return QWEN3_ERR_UNSUPPORTED;
  if (!paged && static_cast<long long>(N) * Hkv * Lmax > 0x7fffffffLL) return QWEN3_ERR_UNSUPPORTED;
  if (!aligned(q, 16) || !aligned(k_new, 16) || !aligned(v_new, 16) || !aligned(k_cache, 16) ||
      !aligned(v_cache, 16) || !aligned(out, 16) || !aligned(q_norm_w, 8) || !aligned(k_norm_w, 8) ||
      !aligned(cache_lens, 4) || (lse != nullptr && !aligned(lse, 4)))
    return QWEN3_ERR_INVALID_ARG;
  if (!(eps >= 0.f)) return QWEN3_ERR_INVALID_ARG;
  return QWEN3_OK;
}

// With `pg`, the cache is paged (k_cache, v_cache unused; Lmax = max_blocks * page).
int decode_impl(const qwen3_bf16* q, const qwen3_bf16* k_new, const qwen3_bf16* v_new, const float* q_norm_w,
                const float* k_norm_w, qwen3_bf16* k_cache, qwen3_bf16* v_cache, const int32_t* cache_lens,
                qwen3_bf16* out, float* lse, int N, int Hq, int Hkv, int d, int Lmax, const Variant& var, float eps,
                void* workspace, size_t ws_bytes, qwen3_stream_t stream, const PagedKV* pg = nullptr) {
  if (pg != nullptr) {
    k_cache = pg->k;
    v_cache = pg->v;
    Lmax = pg->max_blocks * pg->page;
  }
  int st = decode_check(q, k_new, v_new, q_norm_w, k_norm_w, k_cache, v_cache, cache_lens, out, lse, N, Hq, Hkv, d,
                        Lmax, eps, pg != nullptr);
  if (st != QWEN3_OK) return st;
  if (workspace == nullptr || ws_bytes < qwen3_attn_decode_workspace_size(N, Hq, d, Lmax)) return QWEN3_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if ((st = ensure_kernel_attrs()) != QWEN3_OK) return st;

  // 1. Append: normed+rotated k_new and raw v_new into slot L = cache_lens[n].
  st = launch_prologue(k_new, k_norm_w, cache_lens, k_cache, v_new, v_cache, N, 1, Hkv, Lmax, 1, var, eps, s,
                       PrologueQ(), pg, 0);
  if (st != QWEN3_OK) return st;

  // 2. Split-KV attention.
  const int ns = (Lmax + kDecodeSplit - 1) / kDecodeSplit;
  const uintptr_t w0 = (reinterpret_cast<uintptr_t>(workspace) + 255) & ~static_cast<uintptr_t>(255);
  const size_t o_bytes = static_cast<size_t>(N) * Hq * ns * d * 4;
  float* part_o = reinterpret_cast<float*>(w0);
  float* part_lse = reinterpret_cast<float*>((w0 + o_bytes + 255) & ~static_cast<uintptr_t>(255));
  CUtensorMap mk, mv;
  const cuuint64_t rows = pg != nullptr ? static_cast<cuuint64_t>(pg->num_pages) * Hkv * pg->page
                                        : static_cast<cuuint64_t>(N) * Hkv * Lmax;
  // Pages under 64 keys: rows of d viewed as two 64-dim halves, so that one box {64, 2, page}
  // brings a page's keys with both halves.  Otherwise boxes of {64 dims, 64 keys or a page}.
  const bool lines = pg != nullptr && pg->page < 64;
  if (lines) {
    const cuuint64_t dims[3] = {64, 2, rows};
    const cuuint64_t str[2] = {128, kD * 2ull};
    const cuuint32_t box[3] = {64, 2, static_cast<cuuint32_t>(pg->page)};
    if (!make_map(&mk, k_cache, 3, dims, str, box) || !make_map(&mv, v_cache, 3, dims, str, box))
      return QWEN3_ERR_CUDA;
  } else {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(kD), rows};
    const cuuint64_t str[1] = {kD * 2ull};
    const cuuint32_t box[2] = {64, pg != nullptr ? static_cast<cuuint32_t>(std::min(pg->page, 64)) : 64u};
    if (!make_map(&mk, k_cache, 2, dims, str, box) || !make_map(&mv, v_cache, 2, dims, str, box))
      return QWEN3_ERR_CUDA;
  }
  q3::DecodeParams p;
  p.q = reinterpret_cast<const uint32_t*>(q);
  p.q_norm_w = q_norm_w;
  p.cache_lens = cache_lens;
  p.part_o = part_o;
  p.part_lse = part_lse;
  p.N = N;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.log2G = ilog2(Hq / Hkv);
  p.Lmax = Lmax;
  p.split = kDecodeSplit;
  p.n_split_max = ns;
  p.eps = eps;
  p.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(kD)));
  p.wait = next_wait_cfg();
  p.window = var.window;
  p.rope_scale = var.scale;
  p.rope = var.rope;
  p.block_table = pg != nullptr ? pg->table : nullptr;
  p.max_blocks = pg != nullptr ? pg->max_blocks : 0;
  p.log2_page = pg != nullptr ? pg->log2_page : 0;
  p.num_pages = pg != nullptr ? pg->num_pages : 0;
  // Both launches below are programmatic dependent launches (see the kernels): the split
  // kernel overlaps the append, the combine the split kernel's last CTAs.
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(ns, Hkv, N);
  cfg.blockDim = dim3(q3::kDecodeThreads);
  cfg.dynamicSmemBytes = q3::kDecodeSmemBytes;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if ((lines ? cudaLaunchKernelEx(&cfg, q3::decode_split_kernel<true>, mk, mv, p)
             : cudaLaunchKernelEx(&cfg, q3::decode_split_kernel<false>, mk, mv, p)) != cudaSuccess) {
    (void)cudaGetLastError();
    return QWEN3_ERR_CUDA;
  }
  if (cudaGetLastError() != cudaSuccess) return QWEN3_ERR_CUDA;

  // 3. Logsumexp combine of the splits.
  q3::CombineParams c;
  c.part_o = part_o;
  c.part_lse = part_lse;
  c.cache_lens = cache_lens;
  c.out = reinterpret_cast<uint4*>(out);
  c.lse = lse;
  c.Hq = Hq;
  c.Lmax = Lmax;
  c.split = kDecodeSplit;
  c.n_split_max = ns;
  c.window = var.window;
  cfg.gridDim = dim3(N * Hq);
  cfg.blockDim = dim3(128);
  cfg.dynamicSmemBytes = 0;
  if (cudaLaunchKernelEx(&cfg, q3::decode_combine_kernel, c) != cudaSuccess) {
    (void)cudaGetLastError();
    return QWEN3_ERR_CUDA;
  }
  return cudaGetLastError() == cudaSuccess ? QWEN3_OK : QWEN3_ERR_CUDA;
}

}  // namespace

extern "C" {

int qwen3_attn_decode(const qwen3_bf16* q, const qwen3_bf16* k_new, const qwen3_bf16* v_new, const float* q_norm_w,
                      const float* k_norm_w, qwen3_bf16* k_cache, qwen3_bf16* v_cache, const int32_t* cache_lens,
                      qwen3_bf16* out, float* lse, int N, int Hq, int Hkv, int d, int Lmax, float theta, float eps,
                      void* workspace, size_t ws_bytes, qwen3_stream_t stream) {
  NvtxRange nvtx_range("qwen3_attn_decode");
  Variant var;
  const int sv = theta_variant(theta, var);
  if (sv != QWEN3_OK) return sv;
  return decode_impl(q, k_new, v_new, q_norm_w, k_norm_w, k_cache, v_cache, cache_lens, out, lse, N, Hq, Hkv, d,
                     Lmax, var, eps, workspace, ws_bytes, stream);
}

int qwen3_attn_decode_paged(const qwen3_bf16* q, const qwen3_bf16* k_new, const qwen3_bf16* v_new,
                            const float* q_norm_w, const float* k_norm_w, const qwen3_paged_kv* kv,
                            const int32_t* cache_lens, qwen3_bf16* out, float* lse, int N, int Hq, int Hkv, int d,
                            const qwen3_attn_variant* variant, float eps, void* workspace, size_t ws_bytes,
                            qwen3_stream_t stream) {
  NvtxRange nvtx_range("qwen3_attn_decode_paged");
  Variant var;
  int st = make_variant(variant, var);
  if (st != QWEN3_OK) return st;
  if (Hkv <= 0) return QWEN3_ERR_INVALID_ARG;
  PagedKV pg;
  if ((st = make_paged(kv, Hkv, pg)) != QWEN3_OK) return st;
  return decode_impl(q, k_new, v_new, q_norm_w, k_norm_w, nullptr, nullptr, cache_lens, out, lse, N, Hq, Hkv, d, 0,
                     var, eps, workspace, ws_bytes, stream, &pg);
}

int qwen3_attn_prefill_paged(const qwen3_bf16* q, const qwen3_bf16* k, const qwen3_bf16* v, const float* q_norm_w,
                             const float* k_norm_w, const int32_t* pos, qwen3_bf16* out, float* lse,
                             const qwen3_paged_kv* kv, int start, void* workspace, size_t ws_bytes, int B, int T,
                             int Hq, int Hkv, int d, const qwen3_attn_variant* variant, float eps,
                             qwen3_stream_t stream) {
  NvtxRange nvtx_range("qwen3_attn_prefill_paged");
  Variant var;
  int st = make_variant(variant, var);
  if (st != QWEN3_OK) return st;
  if (Hkv <= 0) return QWEN3_ERR_INVALID_ARG;
  PagedKV pg;
  if ((st = make_paged(kv, Hkv, pg)) != QWEN3_OK) return st;
  return prefill_impl(q, k, v, q_norm_w, k_norm_w, pos, out, lse, nullptr, nullptr, start, 0, workspace, ws_bytes, B,
                      T, Hq, Hkv, d, var, eps, stream, &pg);
}

size_t qwen3_qkv_proj_workspace_size(int M) {
  if (M <= 0) return 0;
  return static_cast<size_t>((M + 127) / 128) * 64 * 128 * sizeof(float2) + 256;  // the RoPE table
}

int qwen3_qkv_proj_norm_rope(const qwen3_bf16* x, const qwen3_bf16* w_qkv, const float* q_norm_w,
                             const float* k_norm_w, const int32_t* pos, qwen3_bf16* q_out, qwen3_bf16* k_out,
                             qwen3_bf16* v_out, int M, int hidden, int Hq, int Hkv, int d,
                             const qwen3_attn_variant* variant, float eps, void* workspace, size_t ws_bytes,
                             qwen3_stream_t stream) {
  NvtxRange nvtx_range("qwen3_qkv_proj_norm_rope");
  Variant var;
  int st = make_variant(variant, var);
  if (st != QWEN3_OK) return st;
  if (x == nullptr || w_qkv == nullptr || q_norm_w == nullptr || k_norm_w == nullptr || pos == nullptr ||
      q_out == nullptr || k_out == nullptr || v_out == nullptr)
    return QWEN3_ERR_INVALID_ARG;
  if (M <= 0 || hidden <= 0 || Hq <= 0 || Hkv <= 0) return QWEN3_ERR_INVALID_ARG;
  if (d != kD) return QWEN3_ERR_UNSUPPORTED;
  if (hidden % 8 != 0) return QWEN3_ERR_UNSUPPORTED;  // 16-byte rows for TMA
  if (!aligned(x, 16) || !aligned(w_qkv, 16) || !aligned(q_out, 16) || !aligned(k_out, 16) || !aligned(v_out, 16) ||
      !aligned(q_norm_w, 8) || !aligned(k_norm_w, 8) || !aligned(pos, 4))
    return QWEN3_ERR_INVALID_ARG;
  if (!(eps >= 0.f)) return QWEN3_ERR_INVALID_ARG;
  if (workspace == nullptr || ws_bytes < qwen3_qkv_proj_workspace_size(M)) return QWEN3_ERR_WORKSPACE;
  const int n_heads = Hq + 2 * Hkv;
  if (static_cast<long long>(n_heads) * kD > 0x7fffffffLL || static_cast<long long>(M) * n_heads > 0x7fffffffLL)
    return QWEN3_ERR_UNSUPPORTED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if ((st = ensure_kernel_attrs()) != QWEN3_OK) return st;
  const int n_mt = (M + 127) / 128;
  float2* rope = reinterpret_cast<float2*>((reinterpret_cast<uintptr_t>(workspace) + 255) & ~static_cast<uintptr_t>(255));
  {
    q3::QkvRopeParams rp;
    rp.pos = pos;
    rp.rope = rope;
    rp.M = M;
    rp.n_mt = n_mt;
    rp.scale = var.scale;
    rp.tab = var.rope;
    const long long total = static_cast<long long>(n_mt) * 64 * 128;
    long long blocks = (total + 255) / 256;
    if (blocks > static_cast<long long>(num_sms()) * 32) blocks = static_cast<long long>(num_sms()) * 32;
    q3::qkv_rope_table_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(rp);
    if (cudaGetLastError() != cudaSuccess) return QWEN3_ERR_CUDA;
  }
  q3::QkvParams p;
  p.q_norm_w = q_norm_w;
  p.k_norm_w = k_norm_w;
  p.rope = rope;
  p.q_out = reinterpret_cast<uint4*>(q_out);
  p.k_out = reinterpret_cast<uint4*>(k_out);
  p.v_out = reinterpret_cast<uint4*>(v_out);
  p.M = M;
  p.hidden = hidden;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.n_heads = n_heads;
  p.n_mt = n_mt;
  p.n_nt = (n_heads + 1) / 2;
  const long long n_tiles = static_cast<long long>(p.n_mt) * p.n_nt;
  if (n_tiles > 0x7fffffffLL) return QWEN3_ERR_UNSUPPORTED;
  p.n_tiles = static_cast<int>(n_tiles);
  p.n_k = (hidden + 63) / 64;
  p.eps = eps;
  p.wait = next_wait_cfg();
  // Two SMs per MMA: tiles of 256 tokens (a pair of 128-token tiles) x 256 columns, one
  // cluster of two CTAs per SM pair.  Each SM then loads a third less per K chunk, which
  // pays once a pair's run is long (128 K chunks or more: hidden >= 2048 at 4096 tokens);
  // on shorter runs the one-SM kernel's shorter ring fill and simpler handoffs win.
  p.n_mp = (n_mt + 1) / 2;
  p.n_tiles2 = p.n_mp * p.n_nt;
  const int pairs = num_sms() / 2;
  const long long pair_run = pairs >= 1 ? static_cast<long long>((p.n_tiles2 + pairs - 1) / pairs) * p.n_k : 0;
  int pairs_mode;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    pairs_mode = g_sm_pairs;
  }
  const cuuint64_t xd[2] = {static_cast<cuuint64_t>(hidden), static_cast<cuuint64_t>(M)};
  const cuuint64_t xs[1] = {static_cast<cuuint64_t>(hidden) * 2ull};
  const cuuint32_t xb[2] = {64, 128};
  const cuuint64_t wd[2] = {static_cast<cuuint64_t>(hidden), static_cast<cuuint64_t>(n_heads) * kD};
  CUtensorMap mx, mw;
  if (!make_map(&mx, x, 2, xd, xs, xb)) return QWEN3_ERR_CUDA;
  // The GEMM is a programmatic dependent launch after the RoPE-table kernel: everything
  // before that kernel has completed once it starts, and the GEMM reads the table only
  // after griddep_wait.
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(q3::kQkvThreads);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (pairs >= 1 && pairs_mode != QWEN3_SM_PAIRS_OFF && (pair_run >= 128 || pairs_mode == QWEN3_SM_PAIRS_ALWAYS)) {
    const cuuint32_t wb2[2] = {64, 128};  // each CTA of a pair loads half of a column tile
    if (!make_map(&mw, w_qkv, 2, wd, xs, wb2)) return QWEN3_ERR_CUDA;
    cfg.gridDim = dim3(static_cast<unsigned>(2 * (p.n_tiles2 < pairs ? p.n_tiles2 : pairs)));
    cfg.dynamicSmemBytes = q3::kQkv2SmemBytes;
    if (cudaLaunchKernelEx(&cfg, q3::qkv_proj_pair_kernel, mx, mw, p) == cudaSuccess &&
        cudaGetLastError() == cudaSuccess)
      return QWEN3_OK;
    (void)cudaGetLastError();
  }
  const cuuint32_t wb[2] = {64, 256};
  if (!make_map(&mw, w_qkv, 2, wd, xs, wb)) return QWEN3_ERR_CUDA;
  cfg.gridDim = dim3(static_cast<unsigned>(n_tiles < num_sms() ? n_tiles : num_sms()));
  cfg.dynamicSmemBytes = q3::kQkvSmemBytes;
  if (cudaLaunchKernelEx(&cfg, q3::qkv_proj_kernel, mx, mw, p) != cudaSuccess) {
    (void)cudaGetLastError();
    return QWEN3_ERR_CUDA;
  }
  return cudaGetLastError() == cudaSuccess ? QWEN3_OK : QWEN3_ERR_CUDA;
}

int qwen3_attn_decode_variant(const qwen3_bf16* q, const qwen3_bf16* k_new, const qwen3_bf16* v_new,
                              const float* q_norm_w, const float* k_norm_w, qwen3_bf16* k_cache, qwen3_bf16* v_cache,
                              const int32_t* cache_lens, qwen3_bf16* out, float* lse, int N, int Hq, int Hkv, int d,
                              int Lmax, const qwen3_attn_variant* variant, float eps, void* workspace,
                              size_t ws_bytes, qwen3_stream_t stream) {
  NvtxRange nvtx_range("qwen3_attn_decode_variant");
  Variant var;
  const int sv = make_variant(variant, var);
  if (sv != QWEN3_OK) return sv;
  return decode_impl(q, k_new, v_new, q_norm_w, k_norm_w, k_cache, v_cache, cache_lens, out, lse, N, Hq, Hkv, d,
                     Lmax, var, eps, workspace, ws_bytes, stream);
}

}  // extern "C"

// ---------------------------------------------------------------------------------------
// Decode without any device allocation: the split-KV partials go to a region the library
// declares statically instead of a caller workspace (see qwen3_attn_decode_noalloc in
// include/qwen3_attn.h).  In host code `g_noalloc_scratch` names a host-side stand-in, not
// device memory, so it is never passed to a kernel directly: its device address is looked
// up with cudaGetSymbolAddress while the caller's context is current.
//
// A __device__ variable's address belongs to one CUDA context (the module is loaded into
// each context separately, and again after a device reset recreates the primary context),
// so the address is cached per context, keyed by the driver's context id, which is unique
// for the life of the process and never reused by a later context.
namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[QWEN3_ATTN_NOALLOC_SCRATCH_BYTES];

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// Id of the calling thread's current context; false when there is none (or no driver).
bool current_context_id(unsigned long long* id) {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult r;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &r) == cudaSuccess &&
        r == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &r) == cudaSuccess &&
        r == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
    (void)cudaGetLastError();
  });
  if (get_current == nullptr || get_id == nullptr) return false;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}

constexpr int kNoallocCacheSlots = 64;
std::mutex g_noalloc_mu;
unsigned long long g_noalloc_ctx[kNoallocCacheSlots] = {};
void* g_noalloc_ptr[kNoallocCacheSlots] = {};
int g_noalloc_next = 0;

// Device address of the scratch region in the current context, or nullptr when the lookup
// failed (the runtime's error state is cleared, so the failure does not surface in a later
// call's launch check).
void* noalloc_scratch_for_current_context() {
  unsigned long long id = 0;
  bool have_id = current_context_id(&id);
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (have_id)
    for (int i = 0; i < kNoallocCacheSlots; ++i)
      if (g_noalloc_ptr[i] != nullptr && g_noalloc_ctx[i] == id) return g_noalloc_ptr[i];
  void* ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess) {
    (void)cudaGetLastError();
    return nullptr;
  }
  // the lookup makes the device's primary context current if none was
  if (!have_id) have_id = current_context_id(&id);
  if (have_id) {
    g_noalloc_ctx[g_noalloc_next] = id;
    g_noalloc_ptr[g_noalloc_next] = ptr;
    g_noalloc_next = (g_noalloc_next + 1) % kNoallocCacheSlots;
  }
  return ptr;
}

}  // namespace

extern "C" int qwen3_attn_decode_noalloc(const qwen3_bf16* q, const qwen3_bf16* k_new, const qwen3_bf16* v_new,
                                         const float* q_norm_w, const float* k_norm_w, qwen3_bf16* k_cache,
                                         qwen3_bf16* v_cache, const int32_t* cache_lens, qwen3_bf16* out,
                                         float* lse, int N, int Hq, int Hkv, int d, int Lmax, float theta,
                                         float eps, qwen3_stream_t stream) {
  NvtxRange nvtx_range("qwen3_attn_decode_noalloc");
  // every argument check of qwen3_attn_decode comes before the region's lookup, so a bad
  // argument reports what qwen3_attn_decode reports for it
  Variant var;
  int st = theta_variant(theta, var);
  if (st != QWEN3_OK) return st;
  st = decode_check(q, k_new, v_new, q_norm_w, k_norm_w, k_cache, v_cache, cache_lens, out, lse, N, Hq, Hkv, d, Lmax,
                    eps, false);
  if (st != QWEN3_OK) return st;
  const size_t need = qwen3_attn_decode_workspace_size(N, Hq, d, Lmax);
  if (need > QWEN3_ATTN_NOALLOC_SCRATCH_BYTES) return QWEN3_ERR_WORKSPACE;
  void* scratch = noalloc_scratch_for_current_context();
  if (scratch == nullptr) return QWEN3_ERR_CUDA;
  return qwen3_attn_decode(q, k_new, v_new, q_norm_w, k_norm_w, k_cache, v_cache, cache_lens, out, lse, N, Hq,
                           Hkv, d, Lmax, theta, eps, scratch, QWEN3_ATTN_NOALLOC_SCRATCH_BYTES, stream);
}

// ---------------------------------------------------------------------------------------
// Varlen batches: sequences packed on one token axis, optionally over a paged cache.
namespace {

// Workspace regions of a varlen prefill, each 256-byte aligned: the checked metadata
// (seq [B], the entry list, the item count, rank scratch), Q' [Hkv, N*G, d], and K' and V
// [Hkv, rows, d] with rows = N (fresh prompts: the tokens' own keys) or key_cap (a cache
// in pages under kInPlaceMinPage keys: every sequence's cached and new keys, gathered out of
// the pages; larger pages are read in place and leave these rows unused).
struct VarlenLayout {
  size_t seq = 0, ent = 0, n_items = 0, np = 0, sbase = 0, qp = 0, kp = 0, vp = 0, total = 0;
  int two_p = 0, n_lvl = 0, max_entries = 0;
  long long rows = 0;
};

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

bool varlen_layout(int B, int N, long long key_cap, int Hq, int Hkv, VarlenLayout& L) {
  if (B <= 0 || N <= 0 || key_cap < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || !is_pow2(Hq / Hkv) ||
      Hq / Hkv > 128)
    return false;
  const int G = Hq / Hkv;
  L.two_p = 2 * (128 / G);
  L.n_lvl = (N + L.two_p - 1) / L.two_p;
  const long long max_entries = static_cast<long long>(L.n_lvl) + B;
  if (max_entries * Hkv > 0x7fffffffLL) return false;
  L.max_entries = static_cast<int>(max_entries);
  L.rows = key_cap > 0 ? key_cap : N;  // pages of kInPlaceMinPage keys or more leave these rows unused
  size_t o = 0;
  L.seq = o;
  o = align256(o + static_cast<size_t>(B) * 16);
  L.ent = o;
  o = align256(o + static_cast<size_t>(L.max_entries) * 32);
  L.n_items = o;
  o = align256(o + 4);
  L.np = o;
  o = align256(o + static_cast<size_t>(B) * 4);
  L.sbase = o;
  o = align256(o + static_cast<size_t>(B) * 4);
  L.qp = o;
  o = align256(o + static_cast<size_t>(N) * Hq * kD * 2);
  L.kp = o;
  o = align256(o + static_cast<size_t>(L.rows) * Hkv * kD * 2);
  L.vp = o;
  o = align256(o + static_cast<size_t>(L.rows) * Hkv * kD * 2);
  L.total = o + 256;  // + slack to align the base
  return true;
}

int varlen_impl(const qwen3_bf16* q, const qwen3_bf16* k, const qwen3_bf16* v, const float* q_norm_w,
                const float* k_norm_w, const int32_t* pos, const int32_t* cu, qwen3_bf16* out, float* lse,
                const PagedKV* pg, const int32_t* ctx, long long key_cap, void* workspace, size_t ws_bytes, int B,
                int N, int Hq, int Hkv, int d, const Variant& var, float eps, qwen3_stream_t stream) {
  if (q == nullptr || k == nullptr || v == nullptr || q_norm_w == nullptr || k_norm_w == nullptr || pos == nullptr ||
      cu == nullptr || out == nullptr)
    return QWEN3_ERR_INVALID_ARG;
  if (B <= 0 || N <= 0) return QWEN3_ERR_INVALID_ARG;
  int st = check_common(Hq, Hkv, d);
  if (st != QWEN3_OK) return st;
  if (Hq / Hkv > 128) return QWEN3_ERR_UNSUPPORTED;
  if (pg == nullptr && (ctx != nullptr || key_cap != 0)) return QWEN3_ERR_INVALID_ARG;  // cached keys need a cache
  if (pg != nullptr && key_cap <= 0) return QWEN3_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) || !aligned(q_norm_w, 8) ||
      !aligned(k_norm_w, 8) || !aligned(pos, 4) || !aligned(cu, 4) || (ctx != nullptr && !aligned(ctx, 4)) ||
      (lse != nullptr && !aligned(lse, 4)))
    return QWEN3_ERR_INVALID_ARG;
  if (!(eps >= 0.f)) return QWEN3_ERR_INVALID_ARG;
  // TMA row coordinates and element offsets stay within int32
  if (static_cast<long long>(N) * Hq > (1LL << 31) / kD || key_cap > (1LL << 31) / kD / Hkv ||
      static_cast<long long>(N) * Hkv > (1LL << 31) / kD)
    return QWEN3_ERR_UNSUPPORTED;
  VarlenLayout L;
  if (!varlen_layout(B, N, key_cap, Hq, Hkv, L)) return QWEN3_ERR_UNSUPPORTED;
  if (workspace == nullptr || ws_bytes < L.total) return QWEN3_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if ((st = ensure_kernel_attrs()) != QWEN3_OK) return st;
  const uintptr_t w0 = (reinterpret_cast<uintptr_t>(workspace) + 255) & ~static_cast<uintptr_t>(255);
  int4* seq = reinterpret_cast<int4*>(w0 + L.seq);
  int4* ent = reinterpret_cast<int4*>(w0 + L.ent);
  int* n_items = reinterpret_cast<int*>(w0 + L.n_items);
  qwen3_bf16* qp = reinterpret_cast<qwen3_bf16*>(w0 + L.qp);
  qwen3_bf16* kp = reinterpret_cast<qwen3_bf16*>(w0 + L.kp);
  qwen3_bf16* vp = reinterpret_cast<qwen3_bf16*>(w0 + L.vp);

  // 1. Metadata: checked sequences and the item list, on the device.
  q3::VarlenParams vp_{};
  vp_.cu = cu;
  vp_.ctx = ctx;
  vp_.seq = seq;
  vp_.ent = ent;
  vp_.n_items = n_items;
  vp_.np = reinterpret_cast<int*>(w0 + L.np);
  vp_.sbase = reinterpret_cast<int*>(w0 + L.sbase);
  vp_.key_cap = pg != nullptr ? key_cap : 0;
  vp_.B = B;
  vp_.N = N;
  vp_.two_p = L.two_p;
  vp_.Hkv = Hkv;
  vp_.max_entries = L.max_entries;
  vp_.max_keys = pg != nullptr ? pg->max_blocks * pg->page : 0x7fffffff;
  q3::varlen_setup_kernel<<<1, q3::kVarlenThreads, 0, s>>>(vp_);
  if (cudaGetLastError() != cudaSuccess) return QWEN3_ERR_CUDA;

  // 2. QK prologue over the packed axis (one batch row of N tokens): Q' in the query tiles'
  //    row order; K' and a copy of V into the workspace (fresh prompts) or into each
  //    sequence's pages (a cache).
  PrologueQ pq;
  pq.xq = q;
  pq.wq = q_norm_w;
  pq.dstq = qp;
  pq.Hq = Hq;
  PrologueVarlen vl;
  vl.cu = cu;
  vl.B = B;
  if (pg == nullptr) {
    st = launch_prologue(k, k_norm_w, pos, kp, v, vp, 1, N, Hkv, N, 0, var, eps, s, pq, nullptr, 0, vl);
    if (st != QWEN3_OK) return st;
  } else {
    vl.seq = seq;
    st = launch_prologue(k, k_norm_w, pos, pg->k, v, pg->v, 1, N, Hkv, 1, 0, var, eps, s, pq, pg, 0, vl);
    if (st != QWEN3_OK) return st;
    // 3. The attention kernel reads every sequence's cached and new keys in place, page by
    //    page; pages under kInPlaceMinPage keys are first gathered into the workspace.
    if (pg->page < kInPlaceMinPage) {
      q3::VarlenGatherParams gp{};
      gp.k_pages = reinterpret_cast<const uint4*>(pg->k);
      gp.v_pages = reinterpret_cast<const uint4*>(pg->v);
      gp.block_table = pg->table;
      gp.seq = seq;
      gp.k_out = reinterpret_cast<uint4*>(kp);
      gp.v_out = reinterpret_cast<uint4*>(vp);
      gp.key_cap = key_cap;
      gp.B = B;
      gp.Hkv = Hkv;
      gp.max_blocks = pg->max_blocks;
      gp.log2_page = pg->log2_page;
      gp.num_pages = pg->num_pages;
      const long long chunks = key_cap * Hkv * 16;
      long long blocks = (chunks + 255) / 256;
      if (blocks > static_cast<long long>(num_sms()) * 32) blocks = static_cast<long long>(num_sms()) * 32;
      q3::varlen_gather_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(gp);
      if (cudaGetLastError() != cudaSuccess) return QWEN3_ERR_CUDA;
    }
  }

  // 4. Tensor maps over the packed layouts (batch coordinate 0).
  const int G = Hq / Hkv;
  CUtensorMap mq, mk, mv, mo;
  const cuuint32_t box[4] = {64, 128, 1, 1};
  {
    const cuuint64_t odims[4] = {static_cast<cuuint64_t>(kD), static_cast<cuuint64_t>(Hq),
                                 static_cast<cuuint64_t>(N), 1};
    const cuuint64_t ostr[3] = {kD * 2ull, static_cast<cuuint64_t>(Hq) * kD * 2ull,
                                static_cast<cuuint64_t>(N) * Hq * kD * 2ull};
    const cuuint32_t obox[4] = {64, static_cast<cuuint32_t>(G), static_cast<cuuint32_t>(128 / G), 1};
    if (!make_map(&mo, out, 4, odims, ostr, obox)) return QWEN3_ERR_CUDA;
  }
  {
    const cuuint64_t NG = static_cast<cuuint64_t>(N) * G;
    const cuuint64_t qdims[4] = {static_cast<cuuint64_t>(kD), NG, static_cast<cuuint64_t>(Hkv), 1};
    const cuuint64_t qstr[3] = {kD * 2ull, NG * kD * 2ull, static_cast<cuuint64_t>(Hkv) * NG * kD * 2ull};
    if (!make_map(&mq, qp, 4, qdims, qstr, box)) return QWEN3_ERR_CUDA;
  }
  const bool in_place = pg != nullptr && pg->page >= kInPlaceMinPage;
  if (in_place) {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(kD),
                                static_cast<cuuint64_t>(pg->num_pages) * Hkv * pg->page};
    const cuuint64_t str[1] = {kD * 2ull};
    const cuuint32_t pbox[2] = {64, static_cast<cuuint32_t>(std::min(pg->page, 128))};
    if (!make_map(&mk, pg->k, 2, dims, str, pbox) || !make_map(&mv, pg->v, 2, dims, str, pbox))
      return QWEN3_ERR_CUDA;
  } else {
    const cuuint64_t R = static_cast<cuuint64_t>(L.rows);
    const cuuint64_t dims[4] = {static_cast<cuuint64_t>(kD), R, static_cast<cuuint64_t>(Hkv), 1};
    const cuuint64_t str[3] = {kD * 2ull, R * kD * 2ull, static_cast<cuuint64_t>(Hkv) * R * kD * 2ull};
    if (!make_map(&mk, kp, 4, dims, str, box) || !make_map(&mv, vp, 4, dims, str, box)) return QWEN3_ERR_CUDA;
  }

  // 5. Attention over the device's item list.
  q3::PrefillParams p{};
  p.q_norm_w = q_norm_w;
  p.k_norm_w = k_norm_w;
  p.lse = lse;
  p.B = B;
  p.T = N;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.log2G = ilog2(G);
  p.P = 128 >> p.log2G;
  p.n_items = L.max_entries * Hkv;
  p.start = 0;
  p.window = var.window;
  p.rope_scale = var.scale;
  p.eps = eps;
  p.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(kD)));
  p.wait = next_wait_cfg();
  {
    std::lock_guard<std::mutex> lk(g_mu);
    p.fault = g_fault;
    p.force_rmax = g_softmax_path == QWEN3_SOFTMAX_RUNNING_MAX ? 1 : 0;
  }
  p.vl_ent = ent;
  p.vl_n_items = n_items;
  p.out = reinterpret_cast<uint4*>(out);
  if (in_place) {
    p.block_table = pg->table;
    p.max_blocks = pg->max_blocks;
    p.log2_page = pg->log2_page;
    p.num_pages = pg->num_pages;
  }
  return launch_fmha(mq, mk, mv, mo, p, p.n_items, var.window > 0, true, s);
}

}  // namespace

extern "C" {

size_t qwen3_attn_prefill_varlen_workspace_size(int B, int N, long long key_cap, int Hq, int Hkv, int d) {
  VarlenLayout L;
  if (d != kD || !varlen_layout(B, N, key_cap, Hq, Hkv, L)) return 0;
  return L.total;
}

int qwen3_attn_prefill_varlen(const qwen3_bf16* q, const qwen3_bf16* k, const qwen3_bf16* v, const float* q_norm_w,
                              const float* k_norm_w, const int32_t* pos, const int32_t* cu_seqlens, qwen3_bf16* out,
                              float* lse, const qwen3_paged_kv* kv, const int32_t* ctx_lens, long long key_cap,
                              void* workspace, size_t ws_bytes, int B, int N, int Hq, int Hkv, int d,
                              const qwen3_attn_variant* variant, float eps, qwen3_stream_t stream) {
  NvtxRange nvtx_range("qwen3_attn_prefill_varlen");
  Variant var;
  int st = make_variant(variant, var);
  if (st != QWEN3_OK) return st;
  if (kv == nullptr)
    return varlen_impl(q, k, v, q_norm_w, k_norm_w, pos, cu_seqlens, out, lse, nullptr, ctx_lens, key_cap, workspace,
                       ws_bytes, B, N, Hq, Hkv, d, var, eps, stream);
  if (Hkv <= 0) return QWEN3_ERR_INVALID_ARG;
  PagedKV pg;
  if ((st = make_paged(kv, Hkv, pg)) != QWEN3_OK) return st;
  return varlen_impl(q, k, v, q_norm_w, k_norm_w, pos, cu_seqlens, out, lse, &pg, ctx_lens, key_cap, workspace,
                     ws_bytes, B, N, Hq, Hkv, d, var, eps, stream);
}

}  // extern "C"
