// libmoe_fp4: C ABI of the NVFP4 sparse-MoE layer forward (see include/moe_fp4.h).
//
// Host side: argument checking, device buffers owned by the handle, and the
// launch sequence of one forward:
//   router (+ fp16 staging of x) -> top-k -> permutation / expert classes
//   -> light gate/up + SwiGLU -> light down (x routing weight)
//   -> [dense class on block-scaled FP4 tensor cores] -> combine / unpermute.
// No host synchronisation happens inside moe_fp4_forward; the expert kernels
// read the class lists the permutation kernel left on the device.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <climits>
#include <cstdlib>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <new>

#include "moe_fp4.h"
#include "ptx.cuh"
#include "layout.cuh"
#include "route.cuh"
#include "repack.cuh"
#include "experts.cuh"
#include "combine.cuh"
#include "dense.cuh"
#include "router_tc.cuh"

namespace {

constexpr int kSmallT = 256;          // fused routing kernel up to this many tokens
constexpr size_t kExpSmem1 = moe::expert_smem_size<1>();
constexpr size_t kExpSmem2 = moe::expert_smem_size<2>();
constexpr size_t kExpSmem4 = moe::expert_smem_size<4>();
constexpr int kDenseGridPerSm = 1;
constexpr int kStageEvents = 9;
constexpr int kPermMaxBlocks = 296;       // blocks of the large-batch permutation

struct Workspace {
  void* base = nullptr;
  size_t bytes = 0;
  int max_T = 0;
  float* logits = nullptr;
  int* ids = nullptr;
  float* wts = nullptr;
  int* counts = nullptr;
  int* offsets = nullptr;
  int* perm = nullptr;
  int* inv = nullptr;
  int4* jobs1 = nullptr;
  int* n_jobs1 = nullptr;
  int4* jobs2 = nullptr;
  int* n_jobs2 = nullptr;
  int4* jobs4 = nullptr;
  int* n_jobs4 = nullptr;
  int* counters = nullptr;     // gu_done of the three job lists | exits | ticket
  size_t counter_bytes = 0;
  int4* dense_list = nullptr;
  int* n_dense = nullptr;
  int* dense_ntoff = nullptr;    // [2][E+1]: 128-row and 256-row tile prefixes
  int* perm_bcnt = nullptr;      // [kPermMaxBlocks][E] per-block expert counts / bases
  int* dense_pad_total = nullptr;
  int* act_amax = nullptr;       // [2] max|x|, max|h| bits (dynamic activation scales)
  uint8_t* xq_tok = nullptr;     // dense class: NVFP4 x per token [T][d/2] and scales [T][d/16]
  uint8_t* xsf_tok = nullptr;
  uint8_t* xq = nullptr;         // dense class: NVFP4 activations [pad_rows][d/2]
  uint8_t* xsf = nullptr;        //   and their scale atoms
  uint8_t* hq = nullptr;         // [pad_rows][f/2]
  uint8_t* hsf = nullptr;
  size_t pad_rows = 0;
  CUtensorMap tm_x{}, tm_h{};    // B operands of the dense GEMMs
  // CTA-pair GEMMs: h in 128-row boxes, the x and h scale blocks as byte tensors
  CUtensorMap tm_h2{}, tm_sfx{}, tm_sfh{};
  bool pair_maps = false;
  __nv_bfloat16* rw3 = nullptr;  // router weights split into three exact bf16 parts [3][E][d]
  CUtensorMap tm_rw3{};
  bool tc_router = false;        // tensor-core router available (tensor maps encoded)
  __half* x16 = nullptr;
  float* xscale = nullptr;
  float* h32 = nullptr;
  __half* h16 = nullptr;
  float* partial = nullptr;
  uint16_t* xin = nullptr;     // host-API staging
  uint16_t* xout = nullptr;
};

}  // namespace

struct moe_fp4 {
  int device = 0;
  int E = 0, k = 0, d = 0, f = 0;
  int thr = 9;                    // dense class from 9 rows (measured: the light kernels' 9..32-row jobs
                                  // stream weights slower than the tensor-core class)
  int sm_count = 0;
  int exp_bps1 = 1, exp_bps2 = 1, exp_bps4 = 1;  // resident blocks per SM of the expert kernels
  int64_t wait_timeout_ns = 2000000000LL;
  bool loaded = false;
  uint8_t* gu_frag = nullptr;     // gate/up fragment layout, all experts
  uint8_t* dn_frag = nullptr;     // down fragment layout, all experts
  float* gs = nullptr;            // [3][E]: gate, up, down
  float* l1 = nullptr;            // [2][E]: largest gate / up row L1 norm (expert_l1_kernel)
  int* hexp = nullptr;            // [E]: light-class h staging exponent bound (expert_hexp_kernel)
  bool expert_norm = false;       // RMS-normalise each expert's output before the weighted sum
  bool act_dynamic = false;       // dense class: power-of-two activation tensor scales per call
  bool residual = false;          // out = bf16(x + MoE(x)), the add fused in the combine
  const uint8_t* l2_next = nullptr;   // (set by moe_fp4_forward_layers) prefetched during the experts
  long long l2_next_bytes = 0;
  float norm_eps = 1e-6f;
  int wait_extra = 0;             // test hook: unreachable down-tile completion target
  uint8_t* dq_gu = nullptr;       // dense class: gate/up codes, rows interleaved by 16, signs folded [E*2f][d/2]
  uint8_t* dq_down = nullptr;     // [E*d][f/2]
  uint8_t* dsf_gu = nullptr;      // weight scales, 256-row tile layout (sf_rowpair_offset), rows E*2f, K = d
  uint8_t* dsf_dn = nullptr;      // 128-row tile layout (sf_pair_offset), rows E*d, K = f
  CUtensorMap tm_gu{}, tm_down{};
  // CTA-pair GEMMs: gate/up codes in 128-row boxes, the weight scale blocks as byte tensors
  CUtensorMap tm_gu2{}, tm_sfgu{}, tm_sfdn{};
  bool pair_maps = false;
  int pair_clusters = 0;          // co-resident CTA pairs of the pair GEMM (0: one-CTA GEMMs)
  bool dense_ok = false;          // d, f multiples of 256 and tensor maps available
  bool want_light = true;         // resident weight copies kept by the next load
  bool want_dense = true;
  size_t weight_bytes = 0;        // device bytes of the resident weight copies
  bool dense_h32 = false;         // write fp32 h of the dense class (debug copies)
  int* err = nullptr;             // device error word
  cudaEvent_t stage_ev[kStageEvents] = {};   // optional stage-timing events (caller-owned)
  bool stage_timing = false;
  Workspace ws;
};

namespace {

// The CUDA error behind the last MOE_FP4_ERR_CUDA of this thread, with the
// source line that met it (moe_fp4_last_error_detail).
thread_local char g_err_detail[256] = "";

int cuda_fail(cudaError_t e, int line) {
  snprintf(g_err_detail, sizeof(g_err_detail), "%s (%s) at moe_fp4.cu:%d", cudaGetErrorName(e),
           cudaGetErrorString(e), line);
  (void)cudaGetLastError();
  return MOE_FP4_ERR_CUDA;
}

#define MOE_CUDA(call)                                  \
  do {                                                  \
    cudaError_t e_ = (call);                            \
    if (e_ != cudaSuccess) return cuda_fail(e_, __LINE__); \
  } while (0)

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

template <typename T>
T* carve(uint8_t*& cur, size_t count) {
  T* p = reinterpret_cast<T*>(cur);
  cur += align_up(count * sizeof(T), 256);
  return p;
}

// Largest job list of 17..32-row jobs: every light expert's full 32-row
// jobs plus one remainder each.
size_t max_jobs4(const moe_fp4* h, int Tm) { return (size_t)h->E + (size_t)Tm * h->k / moe::kJobRows + 1; }

// completion counters: gu_done of list 1 [E] | of list 2 [E] | of list 4
// [max_jobs4] | exit 1 | exit 2 | exit 4 | routing ticket
size_t counter_ints(const moe_fp4* h, int Tm) { return (size_t)2 * h->E + max_jobs4(h, Tm) + 4; }

// rows of the dense-class operand buffers: every pair plus up to 127 padding
// rows per dense expert, in whole 128-row tiles
size_t dense_pad_rows(const moe_fp4* h, int Tm) {
  const size_t P = (size_t)Tm * h->k;
  return (P + 256 * std::min<size_t>(h->E, P) + 255) / 256 * 256;
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                   CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                   CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
    else
      (void)cudaGetLastError();
  }
  return fn;
}

// 2-D row-major tensor [rows][row_bytes]; boxes of 128 bytes x box_rows with
// the 128-byte swizzle the tcgen05 K-major shared-memory descriptors expect.
// Rows past `rows` read as zeros.
bool make_map_2d(CUtensorMap* m, const void* base, CUtensorMapDataType dt, uint32_t elem_bytes,
                 uint64_t row_bytes, uint64_t rows, uint32_t box_rows, uint32_t box_bytes = 128) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {row_bytes / elem_bytes, rows};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_bytes / elem_bytes, box_rows};
  const cuuint32_t es[2] = {1, 1};
  return fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            box_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Scale blocks of the dense GEMMs as a 2-D byte tensor of 256-byte rows,
// boxes of box_rows rows (no swizzle): a (tile, stage) block of the M-side
// layout is 8 rows, of the N-side layout 16.
bool make_map_sf(CUtensorMap* m, const void* base, size_t bytes, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || bytes % 256) return false;
  const cuuint64_t dims[2] = {256, bytes / 256};
  const cuuint64_t strides[1] = {256};
  const cuuint32_t box[2] = {256, box_rows};
  const cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Byte operand of the dense GEMMs: rows of kDenseRowBytes per pipeline stage.
bool make_map(CUtensorMap* m, const void* base, uint64_t row_bytes, uint64_t rows, uint32_t box_rows) {
  return make_map_2d(m, base, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, row_bytes, rows, box_rows, moe::kDenseRowBytes);
}

size_t workspace_bytes(const moe_fp4* h, int Tm) {
  const size_t P = (size_t)Tm * h->k;
  size_t b = 0;
  auto add = [&](size_t n) { b += align_up(n, 256); };
  add((size_t)Tm * h->E * 4);       // logits
  add((size_t)3 * h->E * h->d * 2); // router weights, three bf16 parts
  add(P * 4);                       // ids
  add(P * 4);                       // wts
  add((size_t)h->E * 4);            // counts
  add((size_t)(h->E + 1) * 4);      // offsets
  add(P * 4);                       // perm
  add(P * 4);                       // inv
  add((size_t)h->E * 16);                              // light jobs, <= 8 rows
  add(4);
  add((size_t)h->E * 16);                              // light jobs, 9..16 rows
  add(4);
  add(max_jobs4(h, Tm) * 16);                          // light jobs, 17..32 rows
  add(4);
  add(counter_ints(h, Tm) * 4);                        // counters
  add(((size_t)h->E + 1) * 8);                         // dense 128- and 256-row tile prefixes
  add((size_t)kPermMaxBlocks * h->E * 4);              // permutation block counts
  add(4);                                              // dense padded rows
  add(8);                                              // activation amax slots
  const size_t pr = dense_pad_rows(h, Tm);
  add((size_t)Tm * h->d / 2);                          // xq_tok
  add((size_t)Tm * h->d / 16);                         // xsf_tok
  add(pr * h->d / 2);                                  // xq
  add(moe::sf_pair_bytes(pr, h->d));                   // xsf
  add(pr * h->f / 2);                                  // hq
  add(moe::sf_rowpair_bytes(pr, h->f));                // hsf
  add((size_t)h->E * 16);           // dense list
  add(4);
  add((size_t)Tm * h->d * 2);       // x16
  add((size_t)Tm * 4);              // xscale
  add(P * h->f * 4);                // h32
  add(P * h->f * 2);                // h16
  add(P * h->d * 4);                // partial
  add((size_t)Tm * h->d * 2);       // xin
  add((size_t)Tm * h->d * 2);       // xout
  return b;
}

bool make_ws_pair_maps(const moe_fp4* h, Workspace& w) {
  return make_map(&w.tm_h2, w.hq, h->f / 2, w.pad_rows, 128) &&
         make_map_sf(&w.tm_sfx, w.xsf, moe::sf_pair_bytes(w.pad_rows, h->d), 8) &&
         make_map_sf(&w.tm_sfh, w.hsf, moe::sf_rowpair_bytes(w.pad_rows, h->f), 16);
}

int ensure_workspace(moe_fp4* h, int Tm, cudaStream_t stream) {
  if (Tm <= h->ws.max_T && h->ws.base) return MOE_FP4_OK;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(stream, &cs) == cudaSuccess && cs != cudaStreamCaptureStatusNone)
    return MOE_FP4_ERR_CAPTURE;
  if (h->ws.base) {
    MOE_CUDA(cudaDeviceSynchronize());
    cudaFree(h->ws.base);
    h->ws = Workspace{};
  }
  const size_t bytes = workspace_bytes(h, Tm);
  void* base = nullptr;
  if (cudaMalloc(&base, bytes) != cudaSuccess) { (void)cudaGetLastError(); return MOE_FP4_ERR_OOM; }
  Workspace w;
  w.base = base;
  w.bytes = bytes;
  w.max_T = Tm;
  const size_t P = (size_t)Tm * h->k;
  uint8_t* cur = static_cast<uint8_t*>(base);
  w.logits = carve<float>(cur, (size_t)Tm * h->E);
  w.rw3 = carve<__nv_bfloat16>(cur, (size_t)3 * h->E * h->d);
  w.tc_router = make_map_2d(&w.tm_rw3, w.rw3, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)h->d * 2,
                            (uint64_t)3 * h->E, 128);
  w.ids = carve<int>(cur, P);
  w.wts = carve<float>(cur, P);
  w.counts = carve<int>(cur, h->E);
  w.offsets = carve<int>(cur, h->E + 1);
  w.perm = carve<int>(cur, P);
  w.inv = carve<int>(cur, P);
  w.jobs1 = carve<int4>(cur, h->E);
  w.n_jobs1 = carve<int>(cur, 1);
  w.jobs2 = carve<int4>(cur, h->E);
  w.n_jobs2 = carve<int>(cur, 1);
  w.jobs4 = carve<int4>(cur, max_jobs4(h, Tm));
  w.n_jobs4 = carve<int>(cur, 1);
  w.counter_bytes = counter_ints(h, Tm) * 4;
  w.counters = carve<int>(cur, w.counter_bytes / 4);
  w.dense_list = carve<int4>(cur, h->E);
  w.n_dense = carve<int>(cur, 1);
  w.x16 = carve<__half>(cur, (size_t)Tm * h->d);
  w.xscale = carve<float>(cur, Tm);
  w.h32 = carve<float>(cur, P * h->f);
  w.h16 = carve<__half>(cur, P * h->f);
  w.partial = carve<float>(cur, P * h->d);
  w.xin = carve<uint16_t>(cur, (size_t)Tm * h->d);
  w.xout = carve<uint16_t>(cur, (size_t)Tm * h->d);
  w.dense_ntoff = carve<int>(cur, 2 * (h->E + 1));
  w.perm_bcnt = carve<int>(cur, (size_t)kPermMaxBlocks * h->E);
  w.dense_pad_total = carve<int>(cur, 1);
  w.act_amax = carve<int>(cur, 2);
  w.pad_rows = dense_pad_rows(h, Tm);
  w.xq_tok = carve<uint8_t>(cur, (size_t)Tm * h->d / 2);
  w.xsf_tok = carve<uint8_t>(cur, (size_t)Tm * h->d / 16);
  w.xq = carve<uint8_t>(cur, w.pad_rows * h->d / 2);
  w.xsf = carve<uint8_t>(cur, moe::sf_pair_bytes(w.pad_rows, h->d));
  w.hq = carve<uint8_t>(cur, w.pad_rows * h->f / 2);
  w.hsf = carve<uint8_t>(cur, moe::sf_rowpair_bytes(w.pad_rows, h->f));
  if (!make_map(&w.tm_x, w.xq, h->d / 2, w.pad_rows, 128) || !make_map(&w.tm_h, w.hq, h->f / 2, w.pad_rows, 256))
    h->dense_ok = false;
  w.pair_maps = make_ws_pair_maps(h, w);
  if (cudaMemset(w.counters, 0, w.counter_bytes) != cudaSuccess) {
    (void)cudaGetLastError();
    cudaFree(base);
    return MOE_FP4_ERR_CUDA;
  }
  h->ws = w;
  return MOE_FP4_OK;
}

bool ranges_overlap(const void* a, size_t an, const void* b, size_t bn) {
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
  return a0 < b0 + bn && b0 < a0 + an;
}

template <typename... KArgs, typename... Args>
cudaError_t launch(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                   bool pdl, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// The same with thread-block clusters of cluster_x CTAs along x.
template <typename... KArgs, typename... Args>
cudaError_t launch_cluster(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                           bool pdl, unsigned cluster_x, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cluster_x;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// CTA pairs of a pair-GEMM kernel that fit on the device at once (one CTA per SM).
int pair_clusters_resident(const void* fn, size_t smem, int sm_count) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * (sm_count / 2));
  cfg.blockDim = dim3(moe::kDenseThreads);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, fn, &cfg) != cudaSuccess) {
    (void)cudaGetLastError();
    return 0;
  }
  return std::min(n, sm_count / 2);
}

size_t permute_smem_bytes(int E) { return moe::permute_smem_ints(E) * 4; }

// Experts per routing block: two when one K group of 8 per thread covers d.
int route_epb(int d) { return d <= 8192 ? 2 : 1; }

size_t route_smem_bytes(int E, int d, int T, int k) {
  const size_t P = (size_t)T * k;
  const size_t tail = P <= 32 ? moe::route_small_ids_offset(E, T, k) + 32 : 0;
  return std::max((size_t)route_epb(d) * (d + 32 * 32) * 4, tail * 4);
}

// Largest route_kernel shared memory over every T <= kSmallT.
size_t route_smem_max(int E, int d, int k) {
  return std::max(route_smem_bytes(E, d, kSmallT, k), route_smem_bytes(E, d, std::max(1, 32 / k), k));
}

cudaError_t mark(moe_fp4* h, int i, cudaStream_t st) {
  if (!h->stage_timing) return cudaSuccess;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  cudaError_t e = cudaStreamIsCapturing(st, &cs);
  if (e != cudaSuccess) return e;
  return cudaEventRecordWithFlags(h->stage_ev[i], st,
                                  cs == cudaStreamCaptureStatusActive ? cudaEventRecordExternal
                                                                      : cudaEventRecordDefault);
}

// What a call runs besides the plain forward: routing only (stops after the
// permutation), or rows the caller routed (pre_ids, one expert per row,
// weight 1) whose unweighted expert outputs go to y_rows in row order.
struct RunMode {
  bool route_only = false;
  const int* pre_ids = nullptr;
  float* y_rows = nullptr;
};

int run_forward(moe_fp4* h, const void* x, int T, const float* rw, void* out, cudaStream_t st,
                const RunMode& mode = RunMode()) {
  Workspace& w = h->ws;
  const int E = h->E, k = h->k, d = h->d, f = h->f;
  const uint16_t* xb = static_cast<const uint16_t*>(x);
  const bool pdl = !h->stage_timing;
  MOE_CUDA(mark(h, 0, st));
  int* gu_done1 = w.counters;                  // counter layout of counter_ints
  int* gu_done2 = gu_done1 + E;
  int* gu_done4 = gu_done2 + E;
  int* exit1 = gu_done4 + max_jobs4(h, w.max_T);
  int* exit2 = exit1 + 1;
  int* exit4 = exit2 + 1;
  int* ticket = exit4 + 1;
  moe::PermuteOut po{w.counts, w.offsets, w.perm, w.inv, w.jobs1, w.n_jobs1, w.jobs2, w.n_jobs2,
                     w.jobs4, w.n_jobs4, w.dense_list, w.n_dense, w.dense_ntoff, w.dense_pad_total, h->err};
  // Without the dense class (shape or tensor-map support missing) every
  // expert runs in the light class.  An expert holds at most T rows (one per
  // token), so below T = thr no expert can be dense and its kernels are skipped.
  // with only the dense copy resident every expert runs in the dense class
  const bool light_ok = h->gu_frag != nullptr;
  const int dense_ok = h->dense_ok ? 1 : 0;
  // (routing alone needs no expert classes: every active expert counts as light)
  const int thr = mode.route_only ? INT_MAX : !light_ok ? 1 : h->dense_ok ? h->thr : INT_MAX;
  if (!light_ok && !h->dense_ok && !mode.route_only) return MOE_FP4_ERR_UNSUPPORTED;
  const bool run_dense = h->dense_ok && T >= thr;
  const long long P = (long long)T * k;
  const bool small_path = T <= kSmallT && P <= 32 && !mode.pre_ids;
  if (mode.pre_ids) {
    // 1. rows routed by the caller: ids and unit weights, x staging
    MOE_CUDA(launch(moe::preroute_kernel, dim3(std::min<long long>((P + 255) / 256, 8 * h->sm_count)), dim3(256), 0,
                    st, false, mode.pre_ids, (int)P, E, w.ids, w.wts, w.inv, h->err));
    MOE_CUDA(launch(moe::stage_x_kernel, dim3(std::min(T, 8 * h->sm_count)), dim3(256), 0, st, false,
                    xb, T, d, w.x16, w.xscale, h->err));
    MOE_CUDA(mark(h, 1, st));
  } else if (T <= kSmallT) {
    // 1. router logits and x staging; at most 32 pairs: top-k and the
    // permutation in the same launch
    const int epb = route_epb(d), tail = P <= 32 ? 1 : 0;
    // x staging blocks on the SMs the logit blocks leave free (one
    // 1024-thread block fills an SM), for small batches
    const int nlb = (E + epb - 1) / epb;
    const dim3 rgrid(nlb + (T <= 32 ? std::min(T, std::max(0, h->sm_count - nlb)) : 0));
    const size_t rsm = route_smem_bytes(E, d, T, k);
    if (epb == 2)
      MOE_CUDA(launch(moe::route_kernel<2>, rgrid, dim3(1024), rsm, st, false, xb, rw, T, d, E, k, thr,
                      dense_ok, tail, w.logits, w.x16, w.xscale, w.ids, w.wts, ticket, po));
    else
      MOE_CUDA(launch(moe::route_kernel<1>, rgrid, dim3(1024), rsm, st, false, xb, rw, T, d, E, k, thr,
                      dense_ok, tail, w.logits, w.x16, w.xscale, w.ids, w.wts, ticket, po));
    MOE_CUDA(mark(h, 1, st));
  } else {
    // 1. router logits: fp32 weights split into three exact bf16 parts, then
    // the tensor-core GEMM (x bf16 exact products, fp32 accumulation)
    moe::RouterParams rp{};
    const bool tc = w.tc_router && make_map_2d(&rp.tmX, xb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                                               (uint64_t)d * 2, (uint64_t)T, 128);
    if (tc) {
      MOE_CUDA(launch(moe::router_split_kernel, dim3(4 * h->sm_count), dim3(256), 0, st, false,
                      rw, (long long)E * d, w.rw3));
      rp.tmW = w.tm_rw3;
      rp.T = T; rp.d = d; rp.E = E;
      rp.logits = w.logits;
      rp.err = h->err;
      rp.wait_timeout_ns = h->wait_timeout_ns;
      const int tiles = ((E + 127) / 128) * ((T + 127) / 128);
      MOE_CUDA(launch(moe::router_tc_kernel, dim3(std::min(tiles, h->sm_count)), dim3(moe::kRtThreads),
                      moe::router_tc_smem_size(), st, pdl, rp));
    } else {
      MOE_CUDA(launch(moe::router_tiled_kernel, dim3((T + 63) / 64, (E + 63) / 64), dim3(256), 0, st,
                      false, xb, rw, T, d, E, w.logits));
    }
    MOE_CUDA(launch(moe::stage_x_kernel, dim3(std::min(T, 8 * h->sm_count)), dim3(256), 0, st, false,
                    xb, T, d, w.x16, w.xscale, h->err));
    MOE_CUDA(mark(h, 1, st));
  }
  if (small_path) {
    MOE_CUDA(mark(h, 2, st));
  } else {
    // 2. top-k, a warp per token
    if (!mode.pre_ids)
      MOE_CUDA(launch(moe::topk_kernel, dim3((T + 7) / 8), dim3(256), 0, st, false,
                      (const float*)w.logits, T, E, k, w.ids, w.wts));
    MOE_CUDA(mark(h, 2, st));
    // 3. permutation: per-block counts, one-block scan and classes, placement
    const int nb = (int)std::min<long long>(kPermMaxBlocks, std::max<long long>(1, (P + 1023) / 1024));
    MOE_CUDA(launch(moe::perm_hist_kernel, dim3(nb), dim3(1024), (size_t)E * 4, st, false,
                    (const int*)w.ids, P, E, w.perm_bcnt));
    MOE_CUDA(launch(moe::perm_scan_kernel, dim3(1), dim3(1024), permute_smem_bytes(E), st, false,
                    w.perm_bcnt, nb, E, thr, dense_ok, po));
    MOE_CUDA(launch(moe::perm_place_kernel, dim3(nb), dim3(1024), (size_t)32 * E * 4, st, false,
                    (const int*)w.ids, P, E, (const int*)w.perm_bcnt, po));
  }
  MOE_CUDA(mark(h, 3, st));
  if (mode.route_only) return MOE_FP4_OK;
  // the norm and caller-routed rows need the unweighted expert outputs
  const float* wts_epi = (h->expert_norm || mode.pre_ids) ? nullptr : w.wts;
  // 4-5 (dense class). NVFP4 activations, then the two tensor-core GEMMs
  if (run_dense) {
    const bool dyn = h->act_dynamic;
    // CTA pairs (256 x 256 tiles on two SMs) when requested and the device fits them
    const bool pairs = h->pair_clusters > 0 && h->pair_maps && w.pair_maps;
    const int tok_tile = pairs ? 256 : 128;
    if (dyn) {       // max|x| of the call for the x tensor scale
      MOE_CUDA(cudaMemsetAsync(w.act_amax, 0, 2 * sizeof(int), st));
      MOE_CUDA(launch(moe::amax_bf16_kernel, dim3(std::min<long long>(((long long)T * d / 8 + 255) / 256,
                                                                     8 * h->sm_count)),
                      dim3(256), 0, st, false, xb, (long long)T * d, (const int*)w.n_dense, w.act_amax));
    }
    MOE_CUDA(launch(moe::quant_tok_kernel,
                    dim3((unsigned)std::min<long long>(((long long)T * (d / 16) + 255) / 256, 8LL * h->sm_count)),
                    dim3(256), 0, st,
                    pdl && !dyn, xb, T, d, (const int*)w.n_dense, dyn ? (const int*)w.act_amax : nullptr,
                    w.xq_tok, w.xsf_tok));
    MOE_CUDA(launch(moe::gather_x_dense_kernel, dim3(8 * h->sm_count), dim3(256), 0, st, pdl,
                    (const uint8_t*)w.xq_tok, (const uint8_t*)w.xsf_tok, (const int4*)w.dense_list,
                    (const int*)w.n_dense, (const int*)w.dense_pad_total, (const int*)w.perm, k, d, tok_tile,
                    w.xq, w.xsf));
    MOE_CUDA(mark(h, 4, st));
    moe::DenseParams dp{};
    dp.tmA = w.tm_x;           // tokens: the M side of the MMA
    dp.tmB = h->tm_gu;         // weights: 256-row N tiles
    dp.sfA = w.xsf;
    dp.sfB = h->dsf_gu;
    dp.dense = w.dense_list;
    dp.n_dense = w.n_dense;
    dp.ntoff = w.dense_ntoff;
    dp.wt_per_expert = 2 * f / moe::kDenseN;
    dp.rows_per_expert = 2 * f;
    dp.kstages = d / moe::kDenseKStage;
    dp.kb64 = d / 64;
    dp.d = d;
    dp.f = f;
    dp.topk = k;
    dp.gs = h->gs;
    dp.E = E;
    dp.perm = w.perm;
    dp.wts = wts_epi;
    dp.hq = w.hq;
    dp.hsf = w.hsf;
    dp.h32 = (h->dense_h32 || dyn) ? w.h32 : nullptr;
    dp.x_amax = dyn ? w.act_amax : nullptr;
    dp.h_amax = dyn ? w.act_amax + 1 : nullptr;
    dp.partial = w.partial;
    dp.err = h->err;
    dp.wait_timeout_ns = h->wait_timeout_ns;
    if (pairs) {
      moe::DenseParams dq = dp;
      dq.tmB2 = h->tm_gu2;
      dq.tmSfa = w.tm_sfx;
      dq.tmSfb = h->tm_sfgu;
      dq.ntoff = w.dense_ntoff + (E + 1);      // 256-row token tiles
      dq.wt_per_expert = 2 * f / 256;
      MOE_CUDA(launch_cluster(moe::dense_gemm_pair_kernel<moe::kDenseGateUp>, dim3(2 * h->pair_clusters),
                              dim3(moe::kDenseThreads), moe::dense_pair_smem_size<moe::kDenseGateUp>(), st, pdl,
                              2u, dq));
    } else {
      MOE_CUDA(launch(moe::dense_gemm_kernel<moe::kDenseGateUp>, dim3(h->sm_count * kDenseGridPerSm),
                      dim3(moe::kDenseThreads), moe::dense_smem_size<moe::kDenseGateUp>(E), st, pdl, dp));
    }
    MOE_CUDA(mark(h, 5, st));
    if (dyn)         // NVFP4 h with the h tensor scale, once every gate/up tile is done
      MOE_CUDA(launch(moe::quant_h_dense_kernel, dim3(8 * h->sm_count), dim3(256), 0, st, pdl,
                      (const float*)w.h32, (const int4*)w.dense_list, (const int*)w.n_dense,
                      (const int*)w.dense_pad_total, (const int*)(w.act_amax + 1), f, tok_tile, w.hq, w.hsf));
    moe::DenseParams dp2 = dp;
    dp2.x_amax = nullptr;
    dp2.h_amax = nullptr;
    dp2.h_amax_in = dyn ? w.act_amax + 1 : nullptr;
    dp2.tmA = h->tm_down;       // weights: 128-row M tiles
    dp2.tmB = w.tm_h;           // tokens: 256-row N tiles
    dp2.sfA = h->dsf_dn;
    dp2.sfB = w.hsf;
    dp2.ntoff = w.dense_ntoff + (E + 1);
    dp2.wt_per_expert = d / 128;
    dp2.rows_per_expert = d;
    dp2.kstages = f / moe::kDenseKStage;
    dp2.kb64 = f / 64;
    if (pairs) {
      moe::DenseParams dq2 = dp2;
      dq2.tmB2 = w.tm_h2;
      dq2.tmSfa = h->tm_sfdn;
      dq2.tmSfb = w.tm_sfh;
      dq2.ntoff = w.dense_ntoff + (E + 1);
      dq2.wt_per_expert = d / 256;
      MOE_CUDA(launch_cluster(moe::dense_gemm_pair_kernel<moe::kDenseDown>, dim3(2 * h->pair_clusters),
                              dim3(moe::kDenseThreads), moe::dense_pair_smem_size<moe::kDenseDown>(), st, pdl,
                              2u, dq2));
    } else {
      MOE_CUDA(launch(moe::dense_gemm_kernel<moe::kDenseDown>, dim3(h->sm_count * kDenseGridPerSm),
                      dim3(moe::kDenseThreads), moe::dense_smem_size<moe::kDenseDown>(E), st, pdl, dp2));
    }
  } else {
    MOE_CUDA(mark(h, 4, st));
    MOE_CUDA(mark(h, 5, st));
  }
  MOE_CUDA(mark(h, 6, st));
  // 4-6. light experts: gate/up + SwiGLU, down x routing weight, combine
  moe::ExpertParams ep{};
  ep.gu_frag = h->gu_frag;
  ep.dn_frag = h->dn_frag;
  ep.tpe_gu = f / 8;
  ep.cpt_gu = d / moe::kChunkK;
  ep.tpe_dn = d / 16;
  ep.cpt_dn = f / moe::kChunkK;
  ep.perm = w.perm;
  ep.inv = w.inv;
  ep.topk = k;
  ep.T = T;
  ep.d = d;
  ep.f = f;
  ep.E = E;
  ep.x16 = w.x16;
  ep.xscale = w.xscale;
  ep.h16 = w.h16;
  ep.h32 = w.h32;
  ep.gs = h->gs;
  ep.hexp = h->hexp;
  ep.wts = wts_epi;
  ep.wait_extra = h->wait_extra;
  ep.l2_next = h->l2_next;
  ep.l2_next_bytes = h->l2_next_bytes;
  ep.partial = w.partial;
  ep.err = h->err;
  ep.wait_timeout_ns = h->wait_timeout_ns;
  moe::ExpertParams ep1 = ep, ep2 = ep, ep4 = ep;
  ep1.jobs = w.jobs1; ep1.njobs = w.n_jobs1; ep1.gu_done = gu_done1; ep1.exit_cnt = exit1;
  ep2.jobs = w.jobs2; ep2.njobs = w.n_jobs2; ep2.gu_done = gu_done2; ep2.exit_cnt = exit2;
  ep4.jobs = w.jobs4; ep4.njobs = w.n_jobs4; ep4.gu_done = gu_done4; ep4.exit_cnt = exit4;
  ep2.l2_next = ep4.l2_next = nullptr;      // the first light kernel issues the prefetch
  if (light_ok) {
    MOE_CUDA(launch(moe::expert_kernel<1>, dim3(h->sm_count * h->exp_bps1), dim3(moe::kExpThreads),
                    kExpSmem1, st, pdl, ep1));
    // jobs of 9..16 (17..32) rows need a light expert with at least 9 (17)
    // rows: T >= 9 (T >= 17), and a dense threshold above 9 (17) when the
    // dense class runs (every light expert has fewer than thr rows)
    if (T >= 9 && (!run_dense || thr > 9))
      MOE_CUDA(launch(moe::expert_kernel<2>, dim3(h->sm_count * h->exp_bps2), dim3(moe::kExpThreads),
                      kExpSmem2, st, pdl, ep2));
    if (T >= 17 && (!run_dense || thr > 17))
      MOE_CUDA(launch(moe::expert_kernel<4>, dim3(h->sm_count * h->exp_bps4), dim3(moe::kExpThreads),
                      kExpSmem4, st, pdl, ep4));
  }
  MOE_CUDA(mark(h, 7, st));
  // 7. combine / unpermute: out[t] = bf16(sum_j partial[inv[t,j]]), or with
  // the per-expert norm bf16(sum_j w[t,j] * rmsnorm(partial[inv[t,j]]))
  if (mode.pre_ids)
    MOE_CUDA(launch(moe::unpermute_rows_kernel, dim3(std::min<long long>(((long long)T * d / 4 + 255) / 256,
                                                                          8 * h->sm_count)),
                    dim3(256), 0, st, pdl, (const float*)w.partial, (const int*)w.inv, T, d, mode.y_rows));
  else if (h->expert_norm)
    MOE_CUDA(launch(moe::combine_norm_kernel, dim3(std::min(T, 8 * h->sm_count)), dim3(moe::kNormThreads), 0,
                    st, pdl, (const float*)w.partial, (const int*)w.inv, (const float*)w.wts, T, k, d,
                    h->norm_eps, h->residual ? xb : nullptr, static_cast<uint16_t*>(out)));
  else
    MOE_CUDA(launch(moe::combine_kernel, dim3((d + 1023) / 1024, std::min(T, 65535)), dim3(128), 0, st, pdl,
                    (const float*)w.partial, (const int*)w.inv, T, k, d, h->residual ? xb : nullptr,
                    static_cast<uint16_t*>(out)));
  MOE_CUDA(mark(h, 8, st));
  return MOE_FP4_OK;
}

int check_forward_args(moe_fp4* h, const void* x, int T, const float* rw, const void* out) {
  if (!h) return MOE_FP4_ERR_INVALID_ARG;
  if (T < 0) return MOE_FP4_ERR_INVALID_ARG;
  if (T == 0) return MOE_FP4_OK;
  if (!x || !rw || !out) return MOE_FP4_ERR_INVALID_ARG;
  if ((long long)T * h->k >= (1LL << 30)) return MOE_FP4_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(rw) |
       reinterpret_cast<uintptr_t>(out)) & 15)
    return MOE_FP4_ERR_INVALID_ARG;
  const size_t xb = (size_t)T * h->d * 2;
  if (ranges_overlap(x, xb, out, xb)) return MOE_FP4_ERR_INVALID_ARG;
  if (!h->loaded) return MOE_FP4_ERR_NOT_LOADED;
  return MOE_FP4_OK;
}

}  // namespace

extern "C" {

const char* moe_fp4_last_error_detail(void) { return g_err_detail; }

const char* moe_fp4_status_string(int s) {
  switch (s) {
    case MOE_FP4_OK: return "ok";
    case MOE_FP4_ERR_INVALID_ARG: return "invalid argument";
    case MOE_FP4_ERR_UNSUPPORTED: return "unsupported shape or expert class";
    case MOE_FP4_ERR_NOT_LOADED: return "experts not loaded";
    case MOE_FP4_ERR_CUDA: return "CUDA runtime error";
    case MOE_FP4_ERR_OOM: return "device out of memory";
    case MOE_FP4_ERR_DEVICE_TIMEOUT: return "device wait exceeded its bound";
    case MOE_FP4_ERR_NUMERIC: return "fp16 intermediate overflow or non-finite input";
    case MOE_FP4_ERR_CAPTURE: return "workspace growth needed during stream capture";
    default: return "unknown status";
  }
}

int moe_fp4_create(int E, int top_k, int d, int f, moe_fp4_t** out) {
  if (!out) return MOE_FP4_ERR_INVALID_ARG;
  *out = nullptr;
  if (E < 1 || E > 1024) return MOE_FP4_ERR_UNSUPPORTED;
  if (top_k < 1 || top_k > std::min(E, 32)) return MOE_FP4_ERR_UNSUPPORTED;
  if (d < 128 || f < 128 || d > 16384 || f > 16384 || d % 128 || f % 128)
    return MOE_FP4_ERR_UNSUPPORTED;
  moe_fp4* h = new (std::nothrow) moe_fp4();
  if (!h) return MOE_FP4_ERR_OOM;
  h->E = E; h->k = top_k; h->d = d; h->f = f;
  if (const char* s = std::getenv("MOE_FP4_DENSE_THRESHOLD")) {
    const int v = std::atoi(s);
    if (v >= 1) h->thr = v;
  }
  if (const char* s = std::getenv("MOE_FP4_WAIT_TIMEOUT_MS")) {
    const long long v = std::atoll(s);
    if (v >= 1) h->wait_timeout_ns = v * 1000000LL;
  }
  int rc = MOE_FP4_OK;
  do {
    if (cudaGetDevice(&h->device) != cudaSuccess) { rc = MOE_FP4_ERR_CUDA; break; }
    if (cudaDeviceGetAttribute(&h->sm_count, cudaDevAttrMultiProcessorCount, h->device) != cudaSuccess) {
      rc = MOE_FP4_ERR_CUDA; break;
    }
    // The dynamic shared-memory limit is an attribute of the kernel, shared by
    // every handle in the process: only ever raise it, so a handle created
    // later with a smaller shape cannot lower what an earlier one launches.
    auto smem_attr = [](const void* fn, size_t bytes) {
      static std::mutex mu;
      std::lock_guard<std::mutex> lock(mu);
      cudaFuncAttributes fa{};
      cudaError_t e = cudaFuncGetAttributes(&fa, fn);
      if (e != cudaSuccess) return e;
      if ((size_t)fa.maxDynamicSharedSizeBytes >= bytes) return cudaSuccess;
      return cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    };
    if (smem_attr((const void*)moe::expert_kernel<1>, kExpSmem1) != cudaSuccess ||
        smem_attr((const void*)moe::expert_kernel<2>, kExpSmem2) != cudaSuccess ||
        smem_attr((const void*)moe::expert_kernel<4>, kExpSmem4) != cudaSuccess ||
        smem_attr((const void*)moe::perm_scan_kernel, permute_smem_bytes(E)) != cudaSuccess ||
        smem_attr((const void*)moe::perm_place_kernel, (size_t)32 * E * 4) != cudaSuccess ||
        smem_attr((const void*)moe::route_kernel<1>, route_smem_max(E, d, top_k)) != cudaSuccess ||
        smem_attr((const void*)moe::route_kernel<2>, route_smem_max(E, d, top_k)) != cudaSuccess ||
        smem_attr((const void*)moe::dense_gemm_kernel<moe::kDenseGateUp>,
                  moe::dense_smem_size<moe::kDenseGateUp>(E)) != cudaSuccess ||
        smem_attr((const void*)moe::dense_gemm_kernel<moe::kDenseDown>,
                  moe::dense_smem_size<moe::kDenseDown>(E)) != cudaSuccess ||
        smem_attr((const void*)moe::dense_gemm_pair_kernel<moe::kDenseGateUp>,
                  moe::dense_pair_smem_size<moe::kDenseGateUp>()) != cudaSuccess ||
        smem_attr((const void*)moe::dense_gemm_pair_kernel<moe::kDenseDown>,
                  moe::dense_pair_smem_size<moe::kDenseDown>()) != cudaSuccess ||
        smem_attr((const void*)moe::router_tc_kernel, moe::router_tc_smem_size()) != cudaSuccess) {
      rc = MOE_FP4_ERR_CUDA; break;
    }
    // CTA pairs for the dense GEMMs on request (MOE_FP4_DENSE_PAIRS=1): on B200
    // the one-CTA GEMMs measured faster, so they are the default
    {
      const char* ev = std::getenv("MOE_FP4_DENSE_PAIRS");
      const bool want_pairs = ev && ev[0] == '1';
      const int c1 = pair_clusters_resident((const void*)moe::dense_gemm_pair_kernel<moe::kDenseGateUp>,
                                            moe::dense_pair_smem_size<moe::kDenseGateUp>(), h->sm_count);
      const int c2 = pair_clusters_resident((const void*)moe::dense_gemm_pair_kernel<moe::kDenseDown>,
                                            moe::dense_pair_smem_size<moe::kDenseDown>(), h->sm_count);
      h->pair_clusters = want_pairs ? std::min(c1, c2) : 0;
    }
    int nb1 = 0, nb2 = 0, nb4 = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb1, moe::expert_kernel<1>, moe::kExpThreads,
                                                      kExpSmem1) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb2, moe::expert_kernel<2>, moe::kExpThreads,
                                                      kExpSmem2) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb4, moe::expert_kernel<4>, moe::kExpThreads,
                                                      kExpSmem4) != cudaSuccess) {
      rc = MOE_FP4_ERR_CUDA; break;
    }
    h->exp_bps1 = std::max(1, nb1);
    h->exp_bps2 = std::max(1, nb2);
    h->exp_bps4 = std::max(1, nb4);
    if (cudaMalloc(&h->err, sizeof(int)) != cudaSuccess) { rc = MOE_FP4_ERR_OOM; break; }
    if (cudaMemset(h->err, 0, sizeof(int)) != cudaSuccess) { rc = MOE_FP4_ERR_CUDA; break; }
    if (cudaMalloc(&h->gs, sizeof(float) * 3 * E) != cudaSuccess) { rc = MOE_FP4_ERR_OOM; break; }
    if (cudaMalloc(&h->l1, sizeof(float) * 2 * E) != cudaSuccess) { rc = MOE_FP4_ERR_OOM; break; }
    if (cudaMalloc(&h->hexp, sizeof(int) * E) != cudaSuccess) { rc = MOE_FP4_ERR_OOM; break; }
  } while (0);
  if (rc != MOE_FP4_OK) {
    (void)cudaGetLastError();
    moe_fp4_destroy(h);
    return rc;
  }
  *out = h;
  return MOE_FP4_OK;
}

void moe_fp4_destroy(moe_fp4_t* h) {
  if (!h) return;
  cudaDeviceSynchronize();
  cudaFree(h->gu_frag);
  cudaFree(h->dn_frag);
  cudaFree(h->gs);
  cudaFree(h->l1);
  cudaFree(h->hexp);
  cudaFree(h->dq_gu);
  cudaFree(h->dq_down);
  cudaFree(h->dsf_gu);
  cudaFree(h->dsf_dn);
  cudaFree(h->err);
  cudaFree(h->ws.base);
  (void)cudaGetLastError();
  delete h;
}

int moe_fp4_load_experts(moe_fp4_t* h, const moe_fp4_experts* w) {
  if (!h || !w) return MOE_FP4_ERR_INVALID_ARG;
  if (!w->gate_q || !w->gate_sf || !w->gate_gs || !w->up_q || !w->up_sf || !w->up_gs ||
      !w->down_q || !w->down_sf || !w->down_gs)
    return MOE_FP4_ERR_INVALID_ARG;
  const int E = h->E, d = h->d, f = h->f;
  const bool dense_shape = (d % 256 == 0) && (f % 256 == 0);
  if (!h->want_light && !dense_shape) return MOE_FP4_ERR_UNSUPPORTED;
  const size_t gu_bytes = (size_t)E * (f / 8) * (d / moe::kChunkK) * moe::kChunkBytes;
  const size_t dn_bytes = (size_t)E * (d / 16) * (f / moe::kChunkK) * moe::kChunkBytes;
  const size_t gu_codes = (size_t)E * f * d / 2, dn_codes = (size_t)E * d * f / 2;
  const size_t gu_atoms = moe::sf_rowpair_bytes((long long)E * 2 * f, d);
  const size_t dn_atoms = moe::sf_pair_bytes((long long)E * d, f);
  h->loaded = false;
  MOE_CUDA(cudaDeviceSynchronize());
  // copies the caller does not keep are released before anything is allocated
  auto release = [](uint8_t** p) { cudaFree(*p); *p = nullptr; };
  if (!h->want_light) { release(&h->gu_frag); release(&h->dn_frag); }
  if (!h->want_dense || !dense_shape) {
    release(&h->dq_gu); release(&h->dq_down); release(&h->dsf_gu); release(&h->dsf_dn);
    h->dense_ok = false;
  }
  auto alloc = [](uint8_t** p, size_t n) {
    if (*p) return true;
    if (cudaMalloc(p, n) != cudaSuccess) { (void)cudaGetLastError(); *p = nullptr; return false; }
    return true;
  };
  h->weight_bytes = 0;
  if (h->want_light) {
    if (!alloc(&h->gu_frag, gu_bytes) || !alloc(&h->dn_frag, dn_bytes)) return MOE_FP4_ERR_OOM;
    h->weight_bytes += gu_bytes + dn_bytes;
  }
  if (h->want_light) {       // both fragment copies exist only when the light class is kept
    const long long thr_gu = (long long)E * (f / 8) * (d / moe::kChunkK) * 32;
    const int blocks_gu = (int)std::min<long long>((thr_gu + 255) / 256, 65535LL * 16);
    moe::repack_fragment_kernel<moe::kGateUp><<<blocks_gu, 256>>>(w->gate_q, w->gate_sf, w->up_q, w->up_sf,
                                                                 E, f, d, h->gu_frag);
    const long long thr_dn = (long long)E * (d / 16) * (f / moe::kChunkK) * 32;
    const int blocks_dn = (int)std::min<long long>((thr_dn + 255) / 256, 65535LL * 16);
    moe::repack_fragment_kernel<moe::kDown><<<blocks_dn, 256>>>(w->down_q, w->down_sf, nullptr, nullptr,
                                                               E, d, f, h->dn_frag);
    MOE_CUDA(cudaGetLastError());
  }
  // dense class: codes with block-scale signs folded, scale atoms, tensor maps
  if (h->want_dense && dense_shape) {
    if (!alloc(&h->dq_gu, 2 * gu_codes) || !alloc(&h->dq_down, dn_codes) ||
        !alloc(&h->dsf_gu, gu_atoms) || !alloc(&h->dsf_dn, dn_atoms))
      return MOE_FP4_ERR_OOM;
    h->weight_bytes += 2 * gu_codes + dn_codes + gu_atoms + dn_atoms;
    const int blocks = h->sm_count * 8;
    moe::dense_gu_codes_kernel<<<blocks, 256>>>(w->gate_q, w->gate_sf, w->up_q, w->up_sf, E, f, d, h->dq_gu);
    moe::dense_codes_kernel<<<blocks, 256>>>(w->down_q, w->down_sf, (long long)E * d, f, h->dq_down);
    moe::dense_sf_atoms_kernel<moe::kGateUp><<<blocks, 256>>>(w->gate_sf, w->up_sf, E, f, d, h->dsf_gu);
    moe::dense_sf_atoms_kernel<moe::kDown><<<blocks, 256>>>(w->down_sf, nullptr, E, d, f, h->dsf_dn);
    MOE_CUDA(cudaGetLastError());
    h->dense_ok = dense_shape &&
                  make_map(&h->tm_gu, h->dq_gu, d / 2, (uint64_t)E * 2 * f, moe::kDenseN) &&
                  make_map(&h->tm_down, h->dq_down, f / 2, (uint64_t)E * d, 128);
    if (h->ws.base && (!make_map(&h->ws.tm_x, h->ws.xq, d / 2, h->ws.pad_rows, 128) ||
                       !make_map(&h->ws.tm_h, h->ws.hq, f / 2, h->ws.pad_rows, 256)))
      h->dense_ok = false;
    h->pair_maps = make_map(&h->tm_gu2, h->dq_gu, d / 2, (uint64_t)E * 2 * f, 128) &&
                   make_map_sf(&h->tm_sfgu, h->dsf_gu, gu_atoms, 16) &&
                   make_map_sf(&h->tm_sfdn, h->dsf_dn, dn_atoms, 8);
    if (h->ws.base) h->ws.pair_maps = make_ws_pair_maps(h, h->ws);
  }
  MOE_CUDA(cudaMemcpy(h->gs, w->gate_gs, sizeof(float) * E, cudaMemcpyDeviceToDevice));
  MOE_CUDA(cudaMemcpy(h->gs + E, w->up_gs, sizeof(float) * E, cudaMemcpyDeviceToDevice));
  MOE_CUDA(cudaMemcpy(h->gs + 2 * E, w->down_gs, sizeof(float) * E, cudaMemcpyDeviceToDevice));
  // light class: exponent bound of |g| * |u| per expert (h's fp16 staging scale)
  MOE_CUDA(cudaMemset(h->l1, 0, sizeof(float) * 2 * E));
  moe::expert_l1_kernel<<<h->sm_count * 8, 256>>>(w->gate_q, w->gate_sf, w->up_q, w->up_sf, E, f, d, h->l1);
  moe::expert_hexp_kernel<<<(E + 255) / 256, 256>>>(h->l1, h->gs, E, h->hexp);
  MOE_CUDA(cudaGetLastError());
  MOE_CUDA(cudaDeviceSynchronize());
  if (!h->want_light && !h->dense_ok) return MOE_FP4_ERR_UNSUPPORTED;   // tensor maps unavailable
  h->loaded = true;
  return MOE_FP4_OK;
}

int moe_fp4_set_resident_classes(moe_fp4_t* h, int light, int dense) {
  if (!h || (light != 0 && light != 1) || (dense != 0 && dense != 1) || (!light && !dense))
    return MOE_FP4_ERR_INVALID_ARG;
  if (!light && (h->d % 256 || h->f % 256)) return MOE_FP4_ERR_UNSUPPORTED;
  h->want_light = light != 0;
  h->want_dense = dense != 0;
  h->loaded = false;                       // takes effect at the next load
  return MOE_FP4_OK;
}

int moe_fp4_device_bytes(moe_fp4_t* h, size_t* weights, size_t* workspace) {
  if (!h || !weights || !workspace) return MOE_FP4_ERR_INVALID_ARG;
  *weights = h->weight_bytes;
  *workspace = h->ws.bytes;
  return MOE_FP4_OK;
}

int moe_fp4_reserve(moe_fp4_t* h, int max_T) {
  if (!h || max_T < 1) return MOE_FP4_ERR_INVALID_ARG;
  if ((long long)max_T * h->k >= (1LL << 30)) return MOE_FP4_ERR_UNSUPPORTED;
  return ensure_workspace(h, max_T, nullptr);
}

int moe_fp4_set_dense_threshold(moe_fp4_t* h, int thr) {
  if (!h || thr < 1) return MOE_FP4_ERR_INVALID_ARG;
  h->thr = thr;
  return MOE_FP4_OK;
}

int moe_fp4_set_expert_norm(moe_fp4_t* h, int enable, float eps) {
  if (!h || (enable != 0 && enable != 1)) return MOE_FP4_ERR_INVALID_ARG;
  if (enable && !(eps >= 0.f && eps < INFINITY)) return MOE_FP4_ERR_INVALID_ARG;
  if (enable && h->k > moe::kNormMaxK) return MOE_FP4_ERR_UNSUPPORTED;
  h->expert_norm = enable != 0;
  if (enable) h->norm_eps = eps;
  return MOE_FP4_OK;
}

int moe_fp4_set_residual(moe_fp4_t* h, int enable) {
  if (!h || (enable != 0 && enable != 1)) return MOE_FP4_ERR_INVALID_ARG;
  h->residual = enable != 0;
  return MOE_FP4_OK;
}

int moe_fp4_forward_layers(moe_fp4_t* const* layers, int L, const void* x, int T, const float* const* router_w,
                           void* out, cudaStream_t stream) {
  if (!layers || L < 1 || !router_w || T < 0) return MOE_FP4_ERR_INVALID_ARG;
  for (int l = 0; l < L; ++l) {
    if (!layers[l] || !router_w[l]) return MOE_FP4_ERR_INVALID_ARG;
    if (l > 0 && (layers[l] == layers[l - 1] || layers[l]->d != layers[0]->d ||
                  layers[l]->device != layers[0]->device))
      return MOE_FP4_ERR_INVALID_ARG;
  }
  if (T == 0) return MOE_FP4_OK;
  // every check and every workspace first, so nothing runs unless all layers can
  // (x against out for every layer: pointers, alignment, no overlap, loaded)
  for (int l = 0; l < L; ++l) {
    int rc = check_forward_args(layers[l], x, T, router_w[l], out);
    if (rc != MOE_FP4_OK) return rc;
    if ((rc = ensure_workspace(layers[l], T, stream)) != MOE_FP4_OK) return rc;
  }
  // layer l reads layer l-1's output from that handle's staging buffer
  const void* in = x;
  for (int l = 0; l < L; ++l) {
    moe_fp4* h = layers[l];
    void* dst = l == L - 1 ? out : h->ws.xout;
    if (l + 1 < L) {
      h->l2_next = reinterpret_cast<const uint8_t*>(router_w[l + 1]);
      h->l2_next_bytes = (long long)layers[l + 1]->E * layers[l + 1]->d * 4;
    }
    const int rc = run_forward(h, in, T, router_w[l], dst, stream);
    h->l2_next = nullptr;
    h->l2_next_bytes = 0;
    if (rc != MOE_FP4_OK) return rc;
    in = dst;
  }
  return MOE_FP4_OK;
}

int moe_fp4_set_act_scale(moe_fp4_t* h, int dynamic) {
  if (!h || (dynamic != 0 && dynamic != 1)) return MOE_FP4_ERR_INVALID_ARG;
  h->act_dynamic = dynamic != 0;
  return MOE_FP4_OK;
}

int moe_fp4_set_wait_timeout_ms(moe_fp4_t* h, int ms) {
  if (!h || ms < 1) return MOE_FP4_ERR_INVALID_ARG;
  h->wait_timeout_ns = (int64_t)ms * 1000000LL;
  return MOE_FP4_OK;
}

int moe_fp4_set_unreachable_wait(moe_fp4_t* h, int enable) {
  if (!h || (enable != 0 && enable != 1)) return MOE_FP4_ERR_INVALID_ARG;
  h->wait_extra = enable ? (1 << 30) : 0;
  return MOE_FP4_OK;
}

int moe_fp4_forward(moe_fp4_t* h, const void* x, int T, const float* rw, void* out,
                    cudaStream_t stream) {
  int rc = check_forward_args(h, x, T, rw, out);
  if (rc != MOE_FP4_OK || T == 0) return rc;
  rc = ensure_workspace(h, T, stream);
  if (rc != MOE_FP4_OK) return rc;
  return run_forward(h, x, T, rw, out, stream);
}

int moe_fp4_forward_ex(moe_fp4_t* h, const void* x, int T, const float* rw, void* out,
                       cudaStream_t stream, moe_fp4_debug* dbg) {
  if (h) h->dense_h32 = dbg && dbg->h;
  int rc = moe_fp4_forward(h, x, T, rw, out, stream);
  if (h) h->dense_h32 = false;
  if (rc != MOE_FP4_OK || T == 0 || !dbg) return rc;
  const Workspace& w = h->ws;
  const size_t P = (size_t)T * h->k;
  auto cp = [&](void* dst, const void* src, size_t bytes) -> int {
    if (!dst) return MOE_FP4_OK;
    MOE_CUDA(cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToDevice, stream));
    return MOE_FP4_OK;
  };
  if ((rc = cp(dbg->logits, w.logits, (size_t)T * h->E * 4))) return rc;
  if ((rc = cp(dbg->topk_ids, w.ids, P * 4))) return rc;
  if ((rc = cp(dbg->topk_w, w.wts, P * 4))) return rc;
  if ((rc = cp(dbg->counts, w.counts, (size_t)h->E * 4))) return rc;
  if ((rc = cp(dbg->offsets, w.offsets, (size_t)(h->E + 1) * 4))) return rc;
  if ((rc = cp(dbg->perm, w.perm, P * 4))) return rc;
  if ((rc = cp(dbg->h, w.h32, P * h->f * 4))) return rc;
  if ((rc = cp(dbg->partial, w.partial, P * h->d * 4))) return rc;
  return MOE_FP4_OK;
}

int moe_fp4_route(moe_fp4_t* h, const void* x, int T, const float* rw, moe_fp4_routing* r,
                  cudaStream_t stream) {
  if (!h || T < 0 || !r) return MOE_FP4_ERR_INVALID_ARG;
  if (T == 0) return MOE_FP4_OK;
  if (!x || !rw) return MOE_FP4_ERR_INVALID_ARG;
  if ((long long)T * h->k >= (1LL << 30)) return MOE_FP4_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(rw)) & 15) return MOE_FP4_ERR_INVALID_ARG;
  int rc = ensure_workspace(h, T, stream);
  if (rc != MOE_FP4_OK) return rc;
  RunMode mode;
  mode.route_only = true;
  rc = run_forward(h, x, T, rw, nullptr, stream, mode);
  if (rc != MOE_FP4_OK) return rc;
  const Workspace& w = h->ws;
  const size_t P = (size_t)T * h->k;
  auto cp = [&](void* dst, const void* src, size_t bytes) -> int {
    if (!dst) return MOE_FP4_OK;
    MOE_CUDA(cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToDevice, stream));
    return MOE_FP4_OK;
  };
  if ((rc = cp(r->logits, w.logits, (size_t)T * h->E * 4))) return rc;
  if ((rc = cp(r->topk_ids, w.ids, P * 4))) return rc;
  if ((rc = cp(r->topk_w, w.wts, P * 4))) return rc;
  if ((rc = cp(r->counts, w.counts, (size_t)h->E * 4))) return rc;
  if ((rc = cp(r->offsets, w.offsets, (size_t)(h->E + 1) * 4))) return rc;
  if ((rc = cp(r->perm, w.perm, P * 4))) return rc;
  if ((rc = cp(r->inv, w.inv, P * 4))) return rc;
  return MOE_FP4_OK;
}

int moe_fp4_forward_routed(moe_fp4_t* h, const void* rows, int n, const int32_t* expert_ids, float* y_rows,
                           cudaStream_t stream) {
  if (!h || n < 0) return MOE_FP4_ERR_INVALID_ARG;
  if (h->k != 1) return MOE_FP4_ERR_UNSUPPORTED;
  if (n == 0) return MOE_FP4_OK;
  if (!rows || !expert_ids || !y_rows) return MOE_FP4_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(rows) | reinterpret_cast<uintptr_t>(y_rows)) & 15) return MOE_FP4_ERR_INVALID_ARG;
  if (ranges_overlap(rows, (size_t)n * h->d * 2, y_rows, (size_t)n * h->d * 4)) return MOE_FP4_ERR_INVALID_ARG;
  if (!h->loaded) return MOE_FP4_ERR_NOT_LOADED;
  int rc = ensure_workspace(h, n, stream);
  if (rc != MOE_FP4_OK) return rc;
  RunMode mode;
  mode.pre_ids = expert_ids;
  mode.y_rows = y_rows;
  return run_forward(h, rows, n, nullptr, nullptr, stream, mode);
}

int moe_fp4_gather_rows(const void* x, int T, int d, const int32_t* perm, int P, int top_k, void* rows,
                        cudaStream_t stream) {
  if (T < 0 || P < 0 || top_k < 1 || d < 8 || d % 8) return MOE_FP4_ERR_INVALID_ARG;
  if (P == 0) return MOE_FP4_OK;
  if (!x || !perm || !rows || (long long)P > (long long)T * top_k) return MOE_FP4_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(rows)) & 15) return MOE_FP4_ERR_INVALID_ARG;
  int sms = 148;
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  (void)cudaGetLastError();
  const long long chunks = (long long)P * (d / 8);
  MOE_CUDA(launch(moe::gather_rows_kernel, dim3((unsigned)std::min<long long>((chunks + 255) / 256, 8LL * sms)),
                  dim3(256), 0, stream, false, static_cast<const uint16_t*>(x), (const int*)perm, P, top_k, d,
                  static_cast<uint16_t*>(rows)));
  return MOE_FP4_OK;
}

int moe_fp4_combine_rows(const float* y_rows, const int32_t* inv, const float* topk_w, int T, int top_k, int d,
                         void* out, cudaStream_t stream) {
  if (T < 0 || top_k < 1 || d < 8 || d % 8) return MOE_FP4_ERR_INVALID_ARG;
  if (T == 0) return MOE_FP4_OK;
  if (!y_rows || !inv || !topk_w || !out) return MOE_FP4_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(y_rows) | reinterpret_cast<uintptr_t>(out)) & 15) return MOE_FP4_ERR_INVALID_ARG;
  MOE_CUDA(launch(moe::combine_rows_kernel, dim3((d + 1023) / 1024, std::min(T, 65535)), dim3(128), 0, stream,
                  false, y_rows, (const int*)inv, topk_w, T, top_k, d, static_cast<uint16_t*>(out)));
  return MOE_FP4_OK;
}

int moe_fp4_forward_host(moe_fp4_t* h, const void* x_host, int T, const float* rw, void* out_host,
                         cudaStream_t stream) {
  if (!h || T < 0) return MOE_FP4_ERR_INVALID_ARG;
  if (T == 0) return MOE_FP4_OK;
  if (!x_host || !out_host || !rw) return MOE_FP4_ERR_INVALID_ARG;
  if (!h->loaded) return MOE_FP4_ERR_NOT_LOADED;
  int rc = ensure_workspace(h, T, stream);
  if (rc != MOE_FP4_OK) return rc;
  const size_t bytes = (size_t)T * h->d * 2;
  MOE_CUDA(cudaMemcpyAsync(h->ws.xin, x_host, bytes, cudaMemcpyHostToDevice, stream));
  rc = moe_fp4_forward(h, h->ws.xin, T, rw, h->ws.xout, stream);
  if (rc != MOE_FP4_OK) return rc;
  MOE_CUDA(cudaMemcpyAsync(out_host, h->ws.xout, bytes, cudaMemcpyDeviceToHost, stream));
  MOE_CUDA(cudaStreamSynchronize(stream));
  return MOE_FP4_OK;
}

int moe_fp4_set_stage_events(moe_fp4_t* h, cudaEvent_t* events, int n) {
  if (!h) return MOE_FP4_ERR_INVALID_ARG;
  if (n == 0) { h->stage_timing = false; return MOE_FP4_OK; }
  if (n != kStageEvents || !events) return MOE_FP4_ERR_INVALID_ARG;
  for (int i = 0; i < kStageEvents; ++i) {
    if (!events[i]) return MOE_FP4_ERR_INVALID_ARG;
    h->stage_ev[i] = events[i];
  }
  h->stage_timing = true;
  return MOE_FP4_OK;
}

int moe_fp4_get_device_error(moe_fp4_t* h, int* code) {
  if (!h || !code) return MOE_FP4_ERR_INVALID_ARG;
  MOE_CUDA(cudaDeviceSynchronize());
  MOE_CUDA(cudaMemcpy(code, h->err, sizeof(int), cudaMemcpyDeviceToHost));
  MOE_CUDA(cudaMemset(h->err, 0, sizeof(int)));
  // a forward that stopped on an error may leave its completion counters set
  if (*code != MOE_FP4_OK && h->ws.counters)
    MOE_CUDA(cudaMemset(h->ws.counters, 0, h->ws.counter_bytes));
  return MOE_FP4_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free routing (moe_fp4_route_topk_static).
// The logits scratch is a file-scope device array; host code cannot use the
// symbol itself as a device address (in host code it names a host-side
// stand-in), so its device address is looked up once per device, with that
// device current, and passed to the kernels.
// ---------------------------------------------------------------------------
static __device__ __align__(256) float g_route_scratch[MOE_FP4_STATIC_MAX_LOGITS];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
float* g_scratch_ptr[kMaxDevices] = {};

int route_scratch(float** out) {
  int dev = 0;
  MOE_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices) return MOE_FP4_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    MOE_CUDA(cudaGetSymbolAddress(&p, g_route_scratch));
    g_scratch_ptr[dev] = static_cast<float*>(p);
  }
  *out = g_scratch_ptr[dev];
  return MOE_FP4_OK;
}
}  // namespace

extern "C" int moe_fp4_route_topk_static(const void* x_bf16, int T, int d, const float* router_w,
                                         int E, int top_k, int32_t* topk_ids, float* topk_w,
                                         cudaStream_t stream) {
  if (T < 0) return MOE_FP4_ERR_INVALID_ARG;
  if (E < 1 || E > 1024 || top_k < 1 || top_k > std::min(E, 32) || d < 128 || d > 16384 || d % 128)
    return MOE_FP4_ERR_UNSUPPORTED;
  if (T == 0) return MOE_FP4_OK;
  if (!x_bf16 || !router_w || !topk_ids || !topk_w) return MOE_FP4_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(x_bf16) | reinterpret_cast<uintptr_t>(router_w) |
       reinterpret_cast<uintptr_t>(topk_ids) | reinterpret_cast<uintptr_t>(topk_w)) & 15)
    return MOE_FP4_ERR_INVALID_ARG;
  if ((long long)T * E > MOE_FP4_STATIC_MAX_LOGITS) return MOE_FP4_ERR_UNSUPPORTED;
  float* logits = nullptr;
  const int rc = route_scratch(&logits);
  if (rc != MOE_FP4_OK) return rc;
  MOE_CUDA(launch(moe::router_tiled_kernel, dim3((T + 63) / 64, (E + 63) / 64), dim3(256), 0, stream,
                  false, static_cast<const uint16_t*>(x_bf16), router_w, T, d, E, logits));
  MOE_CUDA(launch(moe::topk_kernel, dim3((T + 7) / 8), dim3(256), 0, stream, false,
                  (const float*)logits, T, E, top_k, topk_ids, topk_w));
  return MOE_FP4_OK;
}
