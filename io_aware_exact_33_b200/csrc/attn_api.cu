// attn_api.cu - the C ABI of libattn.so (declared in include/attn.h): host
// argument checks, TMA tensor-map construction, kernel selection and launch.
// Every computation of the attention path runs in the kernels; this file
// only marshals arguments.
#include <algorithm>
#include <climits>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <map>
#include <mutex>
#include <set>
#include <utility>

#include "attn.h"
#include "bwd256_kernel.cuh"
#include "bwd_kernel.cuh"
#include "decode_kernel.cuh"
#include "fwd_fp8_kernel.cuh"
#include "fwd_kernel.cuh"
#include "fwd_persist_kernel.cuh"
#include "merge_kernel.cuh"
#include "sm100.cuh"

namespace {

using namespace attn;

// ------------------------------------------------------------ driver entry
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// (batch, seqlen, heads, headdim) 16-bit tensor as a 4-D TMA map over
// (headdim, heads, seqlen, batch); box = 64 columns x 1 head x `rows` rows,
// 128-byte swizzle.  Rows past seqlen read as zero and are never written.
bool map_bshd(CUtensorMap* m, const void* ptr, bool fp16, int batch, int seqlen, int heads, int d,
              int rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)heads, (cuuint64_t)seqlen, (cuuint64_t)batch};
  cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)heads * d * 2,
                           (cuuint64_t)seqlen * heads * d * 2};
  cuuint32_t box[4] = {64, 1, (cuuint32_t)rows, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(m, fp16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4,
                   const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 8-bit (batch, seqlen, heads, 128) tensor of E4M3 codes as a 4-D map with a
// box of 128 columns (one 128-byte swizzled row) x 1 head x `rows` rows.
bool map_bshd_u8(CUtensorMap* m, const void* ptr, int batch, int seqlen, int heads, int d,
                 int rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)heads, (cuuint64_t)seqlen, (cuuint64_t)batch};
  cuuint64_t strides[3] = {(cuuint64_t)d, (cuuint64_t)heads * d, (cuuint64_t)seqlen * heads * d};
  cuuint32_t box[4] = {128, 1, (cuuint32_t)rows, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void*>(ptr), dims, strides, box,
                   estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// fp32 (batch, seqlen, heads, headdim) tensor as a 4-D map with a box of
// 32 columns x 1 head x 32 rows and 128-byte swizzle (the dQ accumulator).
bool map_bshd_f32_32x32(CUtensorMap* m, const void* ptr, int batch, int seqlen, int heads, int d) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)heads, (cuuint64_t)seqlen, (cuuint64_t)batch};
  cuuint64_t strides[3] = {(cuuint64_t)d * 4, (cuuint64_t)heads * d * 4,
                           (cuuint64_t)seqlen * heads * d * 4};
  cuuint32_t box[4] = {32, 1, 32, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, const_cast<void*>(ptr), dims, strides, box,
                   estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 2-D fp32 map over (cols, rows_total) with box (box_cols, 1), no swizzle.
bool map_f32_rows(CUtensorMap* m, const void* ptr, long long cols, long long rows, int box_cols) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)cols * 4};
  cuuint32_t box[2] = {(cuuint32_t)box_cols, 1};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(ptr), dims, strides, box,
                   estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// bf16 statistics slab (rows_total, nq_pad, kSlabCols) as a 3-D map with a
// box of kSlabCols columns (32 bytes) x `box_rows` rows x 1 and 32-byte
// swizzle, the layout the main kernel's statistics MMA step reads.
bool map_slab(CUtensorMap* m, const void* ptr, long long nq_pad, long long rows, int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)kSlabCols, (cuuint64_t)nq_pad, (cuuint64_t)rows};
  cuuint64_t strides[2] = {(cuuint64_t)kSlabRowBytes, (cuuint64_t)nq_pad * kSlabRowBytes};
  cuuint32_t box[3] = {(cuuint32_t)kSlabCols, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_32B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Opt a kernel into its dynamic shared memory once per (kernel, device).
bool ensure_smem(const void* kernel, int bytes) {
  static std::mutex mu;
  static std::set<std::pair<const void*, int>> done;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  std::lock_guard<std::mutex> g(mu);
  if (done.count({kernel, dev})) return true;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
      cudaSuccess)
    return false;
  done.insert({kernel, dev});
  return true;
}

// Heads per scheduling group (grouped_lpt): as many as keep the tiles they
// share within this share of the 126 MB L2.  16 MB leaves room for what
// streams past them (Q, O, the dQ accumulator): on the causal N=8192
// workload it brought the forward's DRAM reads from 593 MB to 403 MB (Q, K,
// V read once) and the backward's traffic from 1.43 to 1.33 GB, with both
// kernels as fast or faster than at 32 or 64 MB.
constexpr double kL2GroupBudget = 16.0 * 1024 * 1024;
int l2_group(double bytes_per_head, int heads, double budget = kL2GroupBudget) {
  double g = bytes_per_head > 0 ? budget / bytes_per_head : heads;
  if (g < 1) g = 1;
  if (g > heads) g = heads;
  return heads > 0 ? (int)g : 1;
}

bool debug_status_enabled() {
  static int v = -1;
  if (v < 0) {
    const char* e = std::getenv("ATTN_DEBUG_STATUS");
    v = (e && e[0] == '1') ? 1 : 0;
  }
  return v == 1;
}

attn_status finish(cudaStream_t stream) {
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  if (debug_status_enabled()) {
    int code = 0;
    attn_status s = attn_get_device_status(stream, &code);
    if (s != ATTN_OK) return s;
    if (code == ATTN_ERR_TIMEOUT) return ATTN_ERR_TIMEOUT;
    if (code != 0) return ATTN_ERR_DEVICE_STATUS;
  }
  return ATTN_OK;
}

// O = 0 and LSE = -inf for every query when no key exists.
__global__ void fill_empty_fwd(uint16_t* o, long long n_o, float* lse, long long n_lse) {
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n_o; i += stride) o[i] = 0;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n_lse; i += stride)
    lse[i] = -INFINITY;
}

// Zero a 16-bit tensor (gradients of an empty side).
__global__ void fill_zero_u16(uint16_t* x, long long n) {
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += stride) x[i] = 0;
}

int fill_blocks(long long n) {
  long long b = (n + 255) / 256;
  return (int)(b < 1 ? 1 : (b > 4096 ? 4096 : b));
}

// Packed (variable-length) layout of a call: device offsets of the
// sequences and the row counts of the packed tensors.  cu_q == nullptr means
// the dense (batch, seqlen, heads, d) layout.
struct Packed {
  const int* cu_q = nullptr;
  const int* cu_k = nullptr;
  int total_q = 0, total_k = 0;
  bool on() const { return cu_q != nullptr; }
};

// Kernel and grid width of a forward configuration: two query tiles per CTA
// where both O tiles fit tensor memory (d <= 128), one otherwise.
// The one-tile kernel (d = 256) has no dropout variant: attn_check_params
// rejects dropout there before any launch.
template <class C>
struct FwdLaunch {
  template <bool ALIBI, bool DROP>
  static constexpr auto kernel() { return attn_fwd_kernel<C, ALIBI>; }
  static constexpr int rows_per_cta = C::BM;
};
template <int D, int KS, int VS, bool F>
struct FwdLaunch<FwdPPCfg<D, KS, VS, F>> {
  template <bool ALIBI, bool DROP>
  static constexpr auto kernel() {
    return attn_fwd_pp_kernel<FwdPPCfg<D, KS, VS, F>, ALIBI, DROP>;
  }
  static constexpr int rows_per_cta = 2 * FwdPPCfg<D, KS, VS, F>::BM;
};

// Dropout threshold t = round(256 p) of the contract in philox.cuh (0 = no
// dropout); p has been checked to lie in [0, 255.5 / 256).
uint32_t drop_threshold(float p) { return (uint32_t)std::floor(256.0 * (double)p + 0.5); }

// Forward launch.  Dense: p->seqlen_q/k are the lengths.  Packed: p->batch
// sequences of at most p->seqlen_q / p->seqlen_k rows each.
template <class C>
attn_status launch_fwd(const attn_params* p, const void* q, const void* k, const void* v, void* o,
                       float* lse, cudaStream_t stream, const Packed& pk = Packed()) {
  CUtensorMap mq, mk, mv, mo;
  const bool fp16 = C::FP16;
  const int mb = pk.on() ? 1 : p->batch;
  const int nq = pk.on() ? pk.total_q : p->seqlen_q, nk = pk.on() ? pk.total_k : p->seqlen_k;
  if (!map_bshd(&mq, q, fp16, mb, nq, p->nheads, C::D, C::BM) ||
      !map_bshd(&mk, k, fp16, mb, nk, p->nheads_kv, C::D, C::BN) ||
      !map_bshd(&mv, v, fp16, mb, nk, p->nheads_kv, C::D, C::BN) ||
      !map_bshd(&mo, o, fp16, mb, nq, p->nheads, C::D, C::BM))
    return ATTN_ERR_CUDA;
  FwdParams fp;
  fp.cu_q = pk.cu_q;
  fp.cu_k = pk.cu_k;
  fp.total_q = pk.total_q;
  fp.total_k = pk.total_k;
  fp.o = static_cast<uint16_t*>(o);
  fp.alibi = p->alibi_slopes;
  fp.pos_offset = p->pos_offset;
  const uint32_t t = drop_threshold(p->dropout_p);
  fp.drop_seed = p->dropout_seed;
  fp.drop_offset = p->dropout_offset;
  fp.drop_kadd = dropout_kadd(t);
  fp.drop_scale = 256.f / (float)(256u - t);
  fp.lse = lse;
  fp.batch = p->batch;
  fp.nheads = p->nheads;
  fp.nheads_kv = p->nheads_kv;
  fp.seqlen_q = p->seqlen_q;
  fp.seqlen_k = p->seqlen_k;
  fp.causal = p->causal;
  fp.window_left = p->window_left;
  fp.window_right = p->window_right;
  fp.scale_log2 = p->softmax_scale * 1.4426950408889634f;
  fp.num_qblocks = (p->seqlen_q + FwdLaunch<C>::rows_per_cta - 1) / FwdLaunch<C>::rows_per_cta;
  const int heads = p->batch * p->nheads;
  // K and V bytes each query head streams (its kv head's, shared by the group)
  fp.sched_group = l2_group(4.0 * p->seqlen_k * C::D / (p->nheads / p->nheads_kv), heads);
  const long long blocks = (long long)fp.num_qblocks * heads;
  if (blocks > INT_MAX) return ATTN_ERR_INVALID_ARG;
  auto kern = p->alibi_slopes ? (t ? FwdLaunch<C>::template kernel<true, true>()
                                    : FwdLaunch<C>::template kernel<true, false>())
                              : (t ? FwdLaunch<C>::template kernel<false, true>()
                                   : FwdLaunch<C>::template kernel<false, false>());
  if (!ensure_smem(reinterpret_cast<const void*>(kern), C::SMEM_BYTES)) return ATTN_ERR_CUDA;
  kern<<<(unsigned)blocks, C::THREADS, C::SMEM_BYTES, stream>>>(mq, mk, mv, mo, fp);
  return finish(stream);
}

// Mean visible key positions per query row, from the key-tile range of
// each 128-row query tile (the longest sequence's lengths for packed calls).
double mean_visible_keys(const attn_params* p) {
  const long long off = (long long)p->seqlen_k - p->seqlen_q + p->pos_offset;
  const long long kInf = 1ll << 40;
  const long long rb = p->causal ? 0 : (p->window_right >= 0 ? p->window_right : kInf);
  const long long lb = p->window_left >= 0 ? p->window_left : kInf;
  double sum = 0.0;
  long long tiles = 0;
  for (long long q0 = 0; q0 < p->seqlen_q; q0 += 128, ++tiles) {
    const long long q1 = std::min(q0 + 128, (long long)p->seqlen_q) - 1;
    const long long lo = std::max(0ll, q0 + off - lb);
    const long long hi = std::min((long long)p->seqlen_k - 1, q1 + off + rb);
    sum += hi >= lo ? (double)(hi - lo + 1) : 0.0;
  }
  return tiles ? sum / tiles : 0.0;
}

// The persistent forward (fwd_persist_kernel.cuh) for batches of many short
// units, dense or packed: at most 12 key tiles per query tile on average and
// at least four units per SM (packed batches: judged by their longest
// sequence), no positional slopes, no dropout.  On long units the one-shot
// grid measured faster; on the packed mix of 16 causal sequences of
// 256-1792 tokens the persistent kernel measured 0.296 ms against 0.300.
constexpr double kPersistMaxKeys = 12 * 128;
constexpr int kPersistMinUnitsPerSm = 4;
bool use_persistent_fwd(const attn_params* p, const Packed& pk) {
  (void)pk;
  if ((p->headdim != 64 && p->headdim != 128) || p->alibi_slopes ||
      drop_threshold(p->dropout_p) != 0)
    return false;
  int sms = 148, dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long units = ((long long)p->seqlen_q + 255) / 256 * p->batch * p->nheads;
  return units >= (long long)kPersistMinUnitsPerSm * sms &&
         mean_visible_keys(p) <= kPersistMaxKeys;
}

template <class C>
attn_status launch_fwd_persist(const attn_params* p, const void* q, const void* k, const void* v,
                               void* o, float* lse, cudaStream_t stream, const Packed& pk) {
  CUtensorMap mq, mk, mv;
  const int mb = pk.on() ? 1 : p->batch;
  const int nq = pk.on() ? pk.total_q : p->seqlen_q, nk = pk.on() ? pk.total_k : p->seqlen_k;
  if (!map_bshd(&mq, q, C::FP16, mb, nq, p->nheads, C::D, C::BM) ||
      !map_bshd(&mk, k, C::FP16, mb, nk, p->nheads_kv, C::D, C::BN) ||
      !map_bshd(&mv, v, C::FP16, mb, nk, p->nheads_kv, C::D, C::BN))
    return ATTN_ERR_CUDA;
  FwdParams fp;
  std::memset(&fp, 0, sizeof(fp));
  fp.cu_q = pk.cu_q;
  fp.cu_k = pk.cu_k;
  fp.total_q = pk.total_q;
  fp.total_k = pk.total_k;
  fp.o = static_cast<uint16_t*>(o);
  fp.pos_offset = p->pos_offset;
  fp.lse = lse;
  fp.batch = p->batch;
  fp.nheads = p->nheads;
  fp.nheads_kv = p->nheads_kv;
  fp.seqlen_q = p->seqlen_q;
  fp.seqlen_k = p->seqlen_k;
  fp.causal = p->causal;
  fp.window_left = p->window_left;
  fp.window_right = p->window_right;
  fp.scale_log2 = p->softmax_scale * 1.4426950408889634f;
  fp.num_qblocks = (p->seqlen_q + 2 * C::BM - 1) / (2 * C::BM);
  const int heads = p->batch * p->nheads;
  // CTA c takes units c, c + G, ... of the grouped order, which balances
  // best over one long longest-first run: each group restarts it.  Short
  // units mean small per-head K/V, so a 64 MB share still holds a group's
  // (window workload: 0.331 ms against 0.343 ms with the 16 MB groups).
  fp.sched_group = l2_group(4.0 * p->seqlen_k * C::D / (p->nheads / p->nheads_kv), heads,
                            4 * kL2GroupBudget);
  const long long units = (long long)fp.num_qblocks * heads;
  if (units > INT_MAX) return ATTN_ERR_INVALID_ARG;
  int sms = 148, dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = (int)std::min<long long>(units, sms);
  auto kern = attn_fwd_persist_kernel<C>;
  if (!ensure_smem(reinterpret_cast<const void*>(kern), C::SMEM_BYTES)) return ATTN_ERR_CUDA;
  kern<<<grid, C::THREADS, C::SMEM_BYTES, stream>>>(mq, mk, mv, fp, (int)units);
  return finish(stream);
}

// Forward with E4M3 inputs (dense batches, d = 128).
template <class C>
attn_status launch_fwd_e4m3(const attn_params* p, const void* q, const void* k, const void* v,
                            float q_scale, float k_scale, float v_scale, void* o, float* lse,
                            cudaStream_t stream) {
  CUtensorMap mq, mk, mv, mo;
  if (!map_bshd_u8(&mq, q, p->batch, p->seqlen_q, p->nheads, C::D, C::BM) ||
      !map_bshd_u8(&mk, k, p->batch, p->seqlen_k, p->nheads_kv, C::D, C::BN) ||
      !map_bshd_u8(&mv, v, p->batch, p->seqlen_k, p->nheads_kv, C::D, C::BN) ||
      !map_bshd(&mo, o, C::FP16, p->batch, p->seqlen_q, p->nheads, C::D, C::BM))
    return ATTN_ERR_CUDA;
  FwdParams fp;
  std::memset(&fp, 0, sizeof(fp));
  fp.o = static_cast<uint16_t*>(o);
  fp.lse = lse;
  fp.batch = p->batch;
  fp.nheads = p->nheads;
  fp.nheads_kv = p->nheads_kv;
  fp.seqlen_q = p->seqlen_q;
  fp.seqlen_k = p->seqlen_k;
  fp.causal = p->causal;
  fp.window_left = p->window_left;
  fp.window_right = p->window_right;
  fp.pos_offset = p->pos_offset;
  fp.scale_log2 = p->softmax_scale * q_scale * k_scale * 1.4426950408889634f;
  fp.num_qblocks = (p->seqlen_q + 2 * C::BM - 1) / (2 * C::BM);
  const int heads = p->batch * p->nheads;
  // K and V bytes (one per element) each query head streams
  fp.sched_group = l2_group(2.0 * p->seqlen_k * C::D / (p->nheads / p->nheads_kv), heads);
  const long long blocks = (long long)fp.num_qblocks * heads;
  if (blocks > INT_MAX) return ATTN_ERR_INVALID_ARG;
  auto kern = attn_fwd_e4m3_kernel<C>;
  if (!ensure_smem(reinterpret_cast<const void*>(kern), C::SMEM_BYTES)) return ATTN_ERR_CUDA;
  kern<<<(unsigned)blocks, C::THREADS, C::SMEM_BYTES, stream>>>(mq, mk, mv, mo, fp, v_scale);
  return finish(stream);
}

// Key tiles and splits of a decode call: the tiles of kDecodeBN keys from
// the first key any query row sees to the last one, cut into splits so that
// the (batch x kv head x split) blocks fill whole waves of the SMs; cost
// model: waves x (tiles per block + 2 tiles of fixed cost).
struct DecodeSplit {
  int key_lo, tiles_total, splits, tiles_per_split, rmax;
};
DecodeSplit decode_split(const attn_params* p) {
  DecodeSplit d;
  const long long off = (long long)p->seqlen_k - p->seqlen_q;
  const long long kInf = 1ll << 40;
  const long long rb = p->causal ? 0 : (p->window_right >= 0 ? p->window_right : kInf);
  const long long lb = p->window_left >= 0 ? p->window_left : kInf;
  const long long lo = std::max(0ll, off - lb);
  const long long hi = std::min((long long)p->seqlen_k - 1, (long long)p->seqlen_q - 1 + off + rb);
  d.key_lo = (int)std::min(lo, (long long)p->seqlen_k);
  d.tiles_total = hi >= lo ? (int)((hi - lo + kDecodeBN) / kDecodeBN) : 0;
  const int rows = (p->nheads / p->nheads_kv) * p->seqlen_q;
  d.rmax = rows <= 4 ? 4 : (rows <= 8 ? 8 : 16);
  int sms = 148, dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long slots = (long long)sms * (d.rmax <= 8 ? 2 : 1);
  const long long pairs = (long long)p->batch * p->nheads_kv;
  d.splits = 1;
  d.tiles_per_split = std::max(d.tiles_total, 1);
  long long best = -1;
  for (int s = 1; s <= std::min(d.tiles_total, 4096); ++s) {
    const int tps = (d.tiles_total + s - 1) / s;
    const int s_eff = (d.tiles_total + tps - 1) / tps;  // no empty splits
    const long long waves = (pairs * s_eff + slots - 1) / slots;
    const long long cost = waves * (tps + 2);
    if (best < 0 || cost < best) {
      best = cost;
      d.splits = s_eff;
      d.tiles_per_split = tps;
    }
  }
  return d;
}

// Workspace of a decode call: the splits' 16-bit partial outputs, then
// their LSE values.
struct DecodeWorkspace {
  size_t o_bytes, total;
};
DecodeWorkspace decode_layout(const attn_params* p) {
  const size_t rows = (size_t)decode_split(p).splits * p->batch * p->seqlen_q * p->nheads;
  DecodeWorkspace w;
  w.o_bytes = (rows * p->headdim * 2 + 255) / 256 * 256;
  w.total = w.o_bytes + (rows * 4 + 255) / 256 * 256;
  return w;
}

template <int D, bool FP16>
attn_status launch_decode(const attn_params* p, const void* q, const void* k, const void* v,
                          void* o, float* lse, void* workspace, cudaStream_t stream) {
  const DecodeSplit ds = decode_split(p);
  const DecodeWorkspace ws = decode_layout(p);
  CUtensorMap mk, mv;
  if (!map_bshd(&mk, k, FP16, p->batch, p->seqlen_k, p->nheads_kv, D, kDecodeBN) ||
      !map_bshd(&mv, v, FP16, p->batch, p->seqlen_k, p->nheads_kv, D, kDecodeBN))
    return ATTN_ERR_CUDA;
  DecodeParams dp;
  dp.q = static_cast<const uint16_t*>(q);
  dp.o_parts = static_cast<uint16_t*>(workspace);
  dp.lse_parts = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + ws.o_bytes);
  dp.batch = p->batch;
  dp.nheads = p->nheads;
  dp.nheads_kv = p->nheads_kv;
  dp.seqlen_q = p->seqlen_q;
  dp.seqlen_k = p->seqlen_k;
  dp.causal = p->causal;
  dp.window_left = p->window_left;
  dp.window_right = p->window_right;
  dp.scale_log2 = p->softmax_scale * 1.4426950408889634f;
  dp.splits = ds.splits;
  dp.key_lo = ds.key_lo;
  dp.tiles_per_split = ds.tiles_per_split;
  dp.tiles_total = ds.tiles_total;
  auto kern = ds.rmax == 4 ? attn_decode_kernel<D, FP16, 4>
                           : (ds.rmax == 8 ? attn_decode_kernel<D, FP16, 8>
                                           : attn_decode_kernel<D, FP16, 16>);
  if (!ensure_smem(reinterpret_cast<const void*>(kern), DecodeCfg<D>::SMEM_BYTES))
    return ATTN_ERR_CUDA;
  const dim3 grid((unsigned)(p->batch * p->nheads_kv), (unsigned)ds.splits);  // splits <= 4096
  kern<<<grid, kDecodeThreads, DecodeCfg<D>::SMEM_BYTES, stream>>>(mk, mv, dp);
  const attn_status st = finish(stream);
  if (st != ATTN_OK) return st;
  const attn_merge_params mp = {ds.splits, p->batch, p->seqlen_q, p->nheads, p->headdim, p->dtype};
  return attn_merge(&mp, dp.o_parts, dp.lse_parts, o, lse, stream);
}

BwdWorkspace bwd_layout(const attn_params* p, const Packed& pk) {
  return pk.on() ? bwd_workspace_layout_packed(pk.total_q, p->batch, p->nheads, p->headdim)
                 : bwd_workspace_layout(p->batch, p->nheads, p->seqlen_q, p->headdim);
}

BwdParams bwd_params(const attn_params* p, const float* lse, void* workspace, const Packed& pk) {
  const BwdWorkspace ws = bwd_layout(p, pk);
  uint8_t* w = static_cast<uint8_t*>(workspace);
  BwdParams bp;
  bp.cu_q = pk.cu_q;
  bp.cu_k = pk.cu_k;
  bp.total_q = pk.total_q;
  bp.total_k = pk.total_k;
  bp.dk = bp.dv = nullptr;
  bp.acc_f32 = 0;
  bp.alibi = p->alibi_slopes;
  bp.pos_offset = p->pos_offset;
  const uint32_t t = drop_threshold(p->dropout_p);
  bp.drop_seed = p->dropout_seed;
  bp.drop_offset = p->dropout_offset;
  bp.drop_kadd = dropout_kadd(t);
  bp.drop_scale = 256.f / (float)(256u - t);
  bp.num_kblocks = bp.num_qblocks = bp.sched_group = 0;
  bp.lse = lse;
  bp.dvec = reinterpret_cast<float*>(w + ws.dvec_off);
  bp.lse2 = reinterpret_cast<float*>(w + ws.lse2_off);
  bp.lse_slab = reinterpret_cast<uint16_t*>(w + ws.lsb_off);
  bp.dvec_slab = reinterpret_cast<uint16_t*>(w + ws.dvb_off);
  // bf16 without dropout, d <= 128: the main kernel folds the statistics
  // into its MMAs (the d = 256 kernels read the fp32 rows)
  bp.fold = (p->dtype == ATTN_BF16 && t == 0 && p->headdim <= 128) ? 1 : 0;
  bp.dq_acc = reinterpret_cast<float*>(w + ws.dq_off);
  bp.batch = p->batch;
  bp.nheads = p->nheads;
  bp.nheads_kv = p->nheads_kv;
  bp.seqlen_q = p->seqlen_q;
  bp.seqlen_k = p->seqlen_k;
  bp.headdim = p->headdim;
  bp.causal = p->causal;
  bp.window_left = p->window_left;
  bp.window_right = p->window_right;
  bp.scale_log2 = p->softmax_scale * 1.4426950408889634f;
  bp.softmax_scale = p->softmax_scale;
  bp.nq_pad = ws.nq_pad;
  return bp;
}

attn_status launch_bwd_prepare(const attn_params* p, const void* o, const float* lse,
                               const void* dout, void* workspace, cudaStream_t stream,
                               const Packed& pk = Packed()) {
  const BwdParams bp = bwd_params(p, lse, workspace, pk);
  const long long n_rows = (long long)(pk.on() ? 1 : p->batch) * p->nheads * bp.nq_pad;
  // elements of the dQ accumulator
  const long long n_elems = (pk.on() ? bp.nq_pad : (long long)p->batch * p->seqlen_q) *
                            p->nheads * p->headdim;
  if (p->dtype == ATTN_FP16)
    bwd_preprocess<true><<<2368, 256, 0, stream>>>(static_cast<const uint16_t*>(o),
                                                    static_cast<const uint16_t*>(dout), bp, n_rows,
                                                    n_elems / 4);
  else
    bwd_preprocess<false><<<2368, 256, 0, stream>>>(static_cast<const uint16_t*>(o),
                                                     static_cast<const uint16_t*>(dout), bp,
                                                     n_rows, n_elems / 4);
  return finish(stream);
}

template <class C>
attn_status launch_bwd_main(const attn_params* p, const void* q, const void* k, const void* v,
                            const void* dout, void* dk, void* dv, void* workspace,
                            cudaStream_t stream, const Packed& pk = Packed(),
                            bool acc_f32 = false) {
  const BwdParams bp = bwd_params(p, nullptr, workspace, pk);
  const bool fp16 = C::FP16;
  const int mb = pk.on() ? 1 : p->batch;
  const int nq = pk.on() ? pk.total_q : p->seqlen_q, nk = pk.on() ? pk.total_k : p->seqlen_k;
  const long long stat_rows = (long long)mb * p->nheads;  // rows of the Dvec / LSE2 arrays
  CUtensorMap mq, mk, mv, mdo, ml, md, mdk, mdv, mdq;
  if (!map_bshd(&mq, q, fp16, mb, nq, p->nheads, C::D, C::BM) ||
      !map_bshd(&mk, k, fp16, mb, nk, p->nheads_kv, C::D, C::BN) ||
      !map_bshd(&mv, v, fp16, mb, nk, p->nheads_kv, C::D, C::BN) ||
      !map_bshd(&mdo, dout, fp16, mb, nq, p->nheads, C::D, C::BM) ||
      !(bp.fold ? map_slab(&ml, bp.lse_slab, bp.nq_pad, stat_rows, C::BM)
                : map_f32_rows(&ml, bp.lse2, bp.nq_pad, stat_rows, C::BM)) ||
      !(bp.fold ? map_slab(&md, bp.dvec_slab, bp.nq_pad, stat_rows, C::BM)
                : map_f32_rows(&md, bp.dvec, bp.nq_pad, stat_rows, C::BM)) ||
      !(acc_f32 ? map_bshd_f32_32x32(&mdk, dk, mb, nk, p->nheads_kv, C::D)
                : map_bshd(&mdk, dk, fp16, mb, nk, p->nheads_kv, C::D, C::BN)) ||
      !(acc_f32 ? map_bshd_f32_32x32(&mdv, dv, mb, nk, p->nheads_kv, C::D)
                : map_bshd(&mdv, dv, fp16, mb, nk, p->nheads_kv, C::D, C::BN)) ||
      !map_bshd_f32_32x32(&mdq, bp.dq_acc, mb, pk.on() ? (int)bp.nq_pad : p->seqlen_q,
                          p->nheads, C::D))
    return ATTN_ERR_CUDA;
  BwdParams bpl = bp;
  bpl.dk = acc_f32 ? nullptr : static_cast<uint16_t*>(dk);
  bpl.dv = acc_f32 ? nullptr : static_cast<uint16_t*>(dv);
  bpl.acc_f32 = acc_f32 ? 1 : 0;
  bpl.num_kblocks = (p->seqlen_k + C::BN - 1) / C::BN;
  const int heads = p->batch * p->nheads_kv;
  // bytes of Q, dO (16-bit) and the fp32 dQ accumulator each kv head's
  // key tiles share: all query heads of its group
  bpl.sched_group = l2_group(8.0 * p->seqlen_q * C::D * (p->nheads / p->nheads_kv), heads);
  const long long blocks = (long long)bpl.num_kblocks * heads;
  if (blocks > INT_MAX) return ATTN_ERR_INVALID_ARG;
  const bool drop = drop_threshold(p->dropout_p) != 0;
  auto kern = p->alibi_slopes ? (drop ? attn_bwd_kernel<C, true, true> : attn_bwd_kernel<C, true, false>)
                              : (drop ? attn_bwd_kernel<C, false, true> : attn_bwd_kernel<C, false, false>);
  if (!ensure_smem(reinterpret_cast<const void*>(kern), C::SMEM_BYTES)) return ATTN_ERR_CUDA;
  kern<<<(unsigned)blocks, C::THREADS, C::SMEM_BYTES, stream>>>(mq, mk, mv, mdo, ml, md, mdk,
                                                                 mdv, mdq, bpl);
  return finish(stream);
}

// d = 256: dV, then dK (key-stationary), then dQ added to the accumulator
// (query-stationary); see bwd256_kernel.cuh.
template <bool FP16>
attn_status launch_bwd256(const attn_params* p, const void* q, const void* k, const void* v,
                          const void* dout, void* dk, void* dv, void* workspace,
                          cudaStream_t stream, const Packed& pk, bool acc_f32) {
  using KvV = Bwd256KvCfg<FP16, false>;
  using KvK = Bwd256KvCfg<FP16, true>;
  using QC = Bwd256QCfg<FP16>;
  BwdParams bp = bwd_params(p, nullptr, workspace, pk);
  const int mb = pk.on() ? 1 : p->batch;
  const int nq = pk.on() ? pk.total_q : p->seqlen_q, nk = pk.on() ? pk.total_k : p->seqlen_k;
  CUtensorMap mq64, mdo64, mk128, mv128, mq128, mdo128, mk64, mv64;
  if (!map_bshd(&mq64, q, FP16, mb, nq, p->nheads, 256, KvV::BM) ||
      !map_bshd(&mdo64, dout, FP16, mb, nq, p->nheads, 256, KvV::BM) ||
      !map_bshd(&mk128, k, FP16, mb, nk, p->nheads_kv, 256, KvV::BN) ||
      !map_bshd(&mv128, v, FP16, mb, nk, p->nheads_kv, 256, KvV::BN) ||
      !map_bshd(&mq128, q, FP16, mb, nq, p->nheads, 256, QC::BM) ||
      !map_bshd(&mdo128, dout, FP16, mb, nq, p->nheads, 256, QC::BM) ||
      !map_bshd(&mk64, k, FP16, mb, nk, p->nheads_kv, 256, QC::BN) ||
      !map_bshd(&mv64, v, FP16, mb, nk, p->nheads_kv, 256, QC::BN))
    return ATTN_ERR_CUDA;
  bp.acc_f32 = acc_f32 ? 1 : 0;
  const int kv_heads = p->batch * p->nheads_kv, q_heads = p->batch * p->nheads;
  const int group = p->nheads / p->nheads_kv;
  bp.num_kblocks = (p->seqlen_k + KvV::BN - 1) / KvV::BN;
  bp.num_qblocks = (p->seqlen_q + QC::BM - 1) / QC::BM;
  const long long kv_blocks = (long long)bp.num_kblocks * kv_heads;
  const long long q_blocks = (long long)bp.num_qblocks * q_heads;
  if (kv_blocks > INT_MAX || q_blocks > INT_MAX) return ATTN_ERR_INVALID_ARG;
  const bool alibi = p->alibi_slopes != nullptr;
  // key-stationary: Q and dO of a kv head's query heads are shared by its
  // key tiles; query-stationary: K and V of a kv head by its query tiles
  BwdParams bkv = bp;
  bkv.sched_group = l2_group(4.0 * p->seqlen_q * 256 * group, kv_heads);
  BwdParams bq = bp;
  bq.sched_group = l2_group(4.0 * p->seqlen_k * 256 / group, q_heads);
  auto kv_v = alibi ? attn_bwd256_kv_kernel<KvV, true> : attn_bwd256_kv_kernel<KvV, false>;
  auto kv_k = alibi ? attn_bwd256_kv_kernel<KvK, true> : attn_bwd256_kv_kernel<KvK, false>;
  auto qk = alibi ? attn_bwd256_q_kernel<QC, true> : attn_bwd256_q_kernel<QC, false>;
  if (!ensure_smem(reinterpret_cast<const void*>(kv_v), KvV::SMEM_BYTES) ||
      !ensure_smem(reinterpret_cast<const void*>(kv_k), KvK::SMEM_BYTES) ||
      !ensure_smem(reinterpret_cast<const void*>(qk), QC::SMEM_BYTES))
    return ATTN_ERR_CUDA;
  kv_v<<<(unsigned)kv_blocks, KvV::THREADS, KvV::SMEM_BYTES, stream>>>(mq64, mk128, mv128, mdo64,
                                                                      bkv, dv);
  kv_k<<<(unsigned)kv_blocks, KvK::THREADS, KvK::SMEM_BYTES, stream>>>(mq64, mk128, mv128, mdo64,
                                                                      bkv, dk);
  qk<<<(unsigned)q_blocks, QC::THREADS, QC::SMEM_BYTES, stream>>>(mq128, mk64, mv64, mdo128, bq);
  return finish(stream);
}

attn_status launch_bwd_finalize(const attn_params* p, void* dq, void* workspace,
                                cudaStream_t stream, const Packed& pk = Packed()) {
  const BwdParams bp = bwd_params(p, nullptr, workspace, pk);
  const long long n_elems = (pk.on() ? (long long)pk.total_q : (long long)p->batch * p->seqlen_q) *
                            p->nheads * p->headdim;
  if (p->dtype == ATTN_FP16)
    bwd_convert<true><<<2368, 256, 0, stream>>>(bp.dq_acc, static_cast<uint16_t*>(dq),
                                                 n_elems / 4, p->softmax_scale, bp);
  else
    bwd_convert<false><<<2368, 256, 0, stream>>>(bp.dq_acc, static_cast<uint16_t*>(dq),
                                                  n_elems / 4, p->softmax_scale, bp);
  return finish(stream);
}

// Shared argument checks of the backward entry points.  Returns ATTN_OK when
// the call has work to do, or sets *done when it is complete without any.
attn_status bwd_common_checks(const attn_params* p, const void* workspace, size_t workspace_bytes,
                              bool* empty) {
  attn_status st = attn_check_params(p, 1);
  if (st != ATTN_OK) return st;
  *empty = p->batch == 0 || p->seqlen_q == 0 || p->seqlen_k == 0;
  if (*empty) return ATTN_OK;
  const BwdWorkspace ws = bwd_workspace_layout(p->batch, p->nheads, p->seqlen_q, p->headdim);
  if (!workspace || workspace_bytes < ws.total) return ATTN_ERR_WORKSPACE_TOO_SMALL;
  if (reinterpret_cast<uintptr_t>(workspace) & 255u) return ATTN_ERR_MISALIGNED;
  return ATTN_OK;
}

}  // namespace

// Scratch of attn_bwd_noalloc: a file-scope device array, so the entry point
// needs no allocation.  Host code must not pass the symbol itself to a kernel
// (on the host it names a stand-in, not device memory); each device's address
// comes from cudaGetSymbolAddress with that device current.
static __device__ __align__(256) unsigned char g_noalloc_scratch[ATTN_NOALLOC_SCRATCH_BYTES];

namespace {

// Device address of g_noalloc_scratch on the current device, looked up once
// per device; nullptr if the lookup fails.
void* noalloc_scratch_address() {
  static std::mutex mu;
  static std::map<int, void*> addr;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
  std::lock_guard<std::mutex> g(mu);
  auto it = addr.find(dev);
  if (it != addr.end()) return it->second;
  void* ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr)
    return nullptr;
  addr[dev] = ptr;
  return ptr;
}


// Kernel choice by head dimension and dtype.
attn_status dispatch_fwd(const attn_params* p, const void* q, const void* k, const void* v,
                         void* o, float* lse, cudaStream_t stream, const Packed& pk) {
  const bool fp16 = p->dtype == ATTN_FP16;
  const bool persist = use_persistent_fwd(p, pk);
  switch (p->headdim) {
    case 64:
      if (persist)
        return fp16 ? launch_fwd_persist<FwdPersistCfg<64, 3, 3, true>>(p, q, k, v, o, lse, stream, pk)
                    : launch_fwd_persist<FwdPersistCfg<64, 3, 3, false>>(p, q, k, v, o, lse, stream, pk);
      return fp16 ? launch_fwd<FwdPPCfg<64, 3, 3, true>>(p, q, k, v, o, lse, stream, pk)
                  : launch_fwd<FwdPPCfg<64, 3, 3, false>>(p, q, k, v, o, lse, stream, pk);
    case 128:
      if (persist)
        return fp16 ? launch_fwd_persist<FwdPersistCfg<128, 3, 2, true>>(p, q, k, v, o, lse, stream, pk)
                    : launch_fwd_persist<FwdPersistCfg<128, 3, 2, false>>(p, q, k, v, o, lse, stream, pk);
      return fp16 ? launch_fwd<FwdPPCfg<128, 3, 2, true>>(p, q, k, v, o, lse, stream, pk)
                  : launch_fwd<FwdPPCfg<128, 3, 2, false>>(p, q, k, v, o, lse, stream, pk);
    case 256:
      return fp16 ? launch_fwd<FwdCfg<256, 64, 3, 2, true>>(p, q, k, v, o, lse, stream, pk)
                  : launch_fwd<FwdCfg<256, 64, 3, 2, false>>(p, q, k, v, o, lse, stream, pk);
    default:
      return ATTN_ERR_UNSUPPORTED_HEADDIM;
  }
}

attn_status dispatch_bwd_main(const attn_params* p, const void* q, const void* k, const void* v,
                              const void* dout, void* dk, void* dv, void* workspace,
                              cudaStream_t stream, const Packed& pk, bool acc_f32 = false) {
  const bool fp16 = p->dtype == ATTN_FP16;
  switch (p->headdim) {
    case 64:
      return fp16 ? launch_bwd_main<BwdCfg<64, true>>(p, q, k, v, dout, dk, dv, workspace, stream,
                                                      pk, acc_f32)
                  : launch_bwd_main<BwdCfg<64, false>>(p, q, k, v, dout, dk, dv, workspace, stream,
                                                       pk, acc_f32);
    case 128:
      return fp16 ? launch_bwd_main<BwdCfg<128, true>>(p, q, k, v, dout, dk, dv, workspace, stream,
                                                       pk, acc_f32)
                  : launch_bwd_main<BwdCfg<128, false>>(p, q, k, v, dout, dk, dv, workspace, stream,
                                                        pk, acc_f32);
    case 256:
      return fp16 ? launch_bwd256<true>(p, q, k, v, dout, dk, dv, workspace, stream, pk, acc_f32)
                  : launch_bwd256<false>(p, q, k, v, dout, dk, dv, workspace, stream, pk, acc_f32);
    default:
      return ATTN_ERR_UNSUPPORTED_HEADDIM;
  }
}

// The dense-layout view of a packed call: `batch` sequences of at most
// max_seqlen rows (the kernels read each one's own length from the offsets).
attn_params packed_view(const attn_varlen_params* v) {
  attn_params p;
  std::memset(&p, 0, sizeof(p));  // pos_offset 0: each sequence is its own problem
  p.batch = v->batch;
  p.seqlen_q = v->max_seqlen_q;
  p.seqlen_k = v->max_seqlen_k;
  p.nheads = v->nheads;
  p.nheads_kv = v->nheads_kv;
  p.headdim = v->headdim;
  p.dtype = v->dtype;
  p.softmax_scale = v->softmax_scale;
  p.causal = v->causal;
  p.window_left = v->window_left;
  p.window_right = v->window_right;
  p.alibi_slopes = v->alibi_slopes;
  p.dropout_p = v->dropout_p;
  p.dropout_offset = v->dropout_offset;
  p.dropout_seed = v->dropout_seed;
  return p;
}

// Self-test of the bounded wait: two waiters (one warp-uniform, one single
// thread) on an mbarrier that nothing ever arrives at.  Both must give up
// after `limit_ns`, record the timeout in the status word, and return.
__global__ void selftest_bounded_wait_kernel(unsigned long long limit_ns, int* result) {
  __shared__ __align__(8) unsigned long long bar_word;
  const uint32_t bar = smem_addr(&bar_word);
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x < 32) {
    const bool ok = mbar_wait_warp(bar, 0, limit_ns);
    if (threadIdx.x == 0 && result) result[0] = ok ? 0 : 1;
  } else if (threadIdx.x == 32) {
    const bool ok = mbar_wait(bar, 0, limit_ns);
    if (result) result[1] = ok ? 0 : 1;
  }
}

}  // namespace

extern "C" {

const char* attn_version(void) { return "0.1.0"; }

const char* attn_status_string(int s) {
  switch (s) {
    case ATTN_OK: return "ok";
    case ATTN_ERR_INVALID_ARG: return "invalid argument";
    case ATTN_ERR_UNSUPPORTED_HEADDIM: return "unsupported head dimension";
    case ATTN_ERR_UNSUPPORTED_DTYPE: return "unsupported dtype (bf16 or fp16 only)";
    case ATTN_ERR_MISALIGNED: return "tensor pointer not 16-byte aligned";
    case ATTN_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case ATTN_ERR_CUDA: return "CUDA call failed";
    case ATTN_ERR_TIMEOUT: return "device-side wait timed out";
    case ATTN_ERR_DEVICE_STATUS: return "device status word holds an error";
    default: return "unknown status";
  }
}

attn_status attn_check_params(const attn_params* p, int pass) {
  if (!p || (pass != 0 && pass != 1)) return ATTN_ERR_INVALID_ARG;
  if (p->batch < 0 || p->seqlen_q < 0 || p->seqlen_k < 0) return ATTN_ERR_INVALID_ARG;
  if (p->nheads <= 0 || p->nheads_kv <= 0 || p->nheads % p->nheads_kv != 0)
    return ATTN_ERR_INVALID_ARG;
  if (p->nheads > 65535 || p->batch > 65535) return ATTN_ERR_INVALID_ARG;
  if (p->dtype != ATTN_BF16 && p->dtype != ATTN_FP16) return ATTN_ERR_UNSUPPORTED_DTYPE;
  const int d = p->headdim;
  if (d != 64 && d != 128 && d != 256) return ATTN_ERR_UNSUPPORTED_HEADDIM;
  if (!(p->softmax_scale > 0.f) || !std::isfinite(p->softmax_scale)) return ATTN_ERR_INVALID_ARG;
  if (p->causal != 0 && p->causal != 1) return ATTN_ERR_INVALID_ARG;
  if (p->window_left < -1 || p->window_right < -1) return ATTN_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(p->alibi_slopes) & 3u) return ATTN_ERR_MISALIGNED;
  if (!(p->dropout_p >= 0.f) || !(p->dropout_p < 1.f) || drop_threshold(p->dropout_p) > 255u)
    return ATTN_ERR_INVALID_ARG;
  if (d == 256 && drop_threshold(p->dropout_p) != 0) return ATTN_ERR_UNSUPPORTED_HEADDIM;
  if (p->reserved0 != 0) return ATTN_ERR_INVALID_ARG;
  return ATTN_OK;
}

attn_status attn_fwd_e4m3(const attn_params* p, const void* q, const void* k, const void* v,
                          float q_scale, float k_scale, float v_scale, void* o, float* lse,
                          void* stream_) {
  attn_status st = attn_check_params(p, 0);
  if (st != ATTN_OK) return st;
  if (p->headdim != 128) return ATTN_ERR_UNSUPPORTED_HEADDIM;
  if (p->alibi_slopes || drop_threshold(p->dropout_p) != 0) return ATTN_ERR_INVALID_ARG;
  for (float sc : {q_scale, k_scale, v_scale})
    if (!(sc > 0.f) || !std::isfinite(sc)) return ATTN_ERR_INVALID_ARG;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (p->batch == 0 || p->seqlen_q == 0) return ATTN_OK;
  if (!o || !lse) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(o) || (reinterpret_cast<uintptr_t>(lse) & 3u)) return ATTN_ERR_MISALIGNED;
  if (p->seqlen_k == 0) {
    const long long n_o = (long long)p->batch * p->seqlen_q * p->nheads * p->headdim;
    const long long n_l = (long long)p->batch * p->nheads * p->seqlen_q;
    fill_empty_fwd<<<fill_blocks(n_o), 256, 0, stream>>>(static_cast<uint16_t*>(o), n_o, lse, n_l);
    return finish(stream);
  }
  if (!q || !k || !v) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v)) return ATTN_ERR_MISALIGNED;
  return p->dtype == ATTN_FP16
             ? launch_fwd_e4m3<FwdF8Cfg<3, 2, true>>(p, q, k, v, q_scale, k_scale, v_scale, o, lse,
                                                     stream)
             : launch_fwd_e4m3<FwdF8Cfg<3, 2, false>>(p, q, k, v, q_scale, k_scale, v_scale, o,
                                                      lse, stream);
}

size_t attn_fwd_decode_workspace_size(const attn_params* p) {
  if (attn_check_params(p, 0) != ATTN_OK) return 0;
  return decode_layout(p).total;
}

attn_status attn_fwd_decode(const attn_params* p, const void* q, const void* k, const void* v,
                            void* o, float* lse, void* workspace, size_t workspace_bytes,
                            void* stream_) {
  attn_status st = attn_check_params(p, 0);
  if (st != ATTN_OK) return st;
  if (p->headdim != 64 && p->headdim != 128) return ATTN_ERR_UNSUPPORTED_HEADDIM;
  if (p->alibi_slopes || drop_threshold(p->dropout_p) != 0 || p->pos_offset != 0)
    return ATTN_ERR_INVALID_ARG;
  if ((long long)(p->nheads / p->nheads_kv) * p->seqlen_q > kDecodeRows) return ATTN_ERR_INVALID_ARG;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (p->batch == 0 || p->seqlen_q == 0) return ATTN_OK;
  if (!o || !lse) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(o) || (reinterpret_cast<uintptr_t>(lse) & 3u)) return ATTN_ERR_MISALIGNED;
  if (p->seqlen_k == 0) {
    const long long n_o = (long long)p->batch * p->seqlen_q * p->nheads * p->headdim;
    const long long n_l = (long long)p->batch * p->nheads * p->seqlen_q;
    fill_empty_fwd<<<fill_blocks(n_o), 256, 0, stream>>>(static_cast<uint16_t*>(o), n_o, lse, n_l);
    return finish(stream);
  }
  if (!q || !k || !v || !workspace) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return ATTN_ERR_MISALIGNED;
  if (workspace_bytes < decode_layout(p).total) return ATTN_ERR_WORKSPACE_TOO_SMALL;
  const bool fp16 = p->dtype == ATTN_FP16;
  if (p->headdim == 64)
    return fp16 ? launch_decode<64, true>(p, q, k, v, o, lse, workspace, stream)
                : launch_decode<64, false>(p, q, k, v, o, lse, workspace, stream);
  return fp16 ? launch_decode<128, true>(p, q, k, v, o, lse, workspace, stream)
              : launch_decode<128, false>(p, q, k, v, o, lse, workspace, stream);
}

size_t attn_fwd_workspace_size(const attn_params* p) {
  (void)p;
  return 0;
}

attn_status attn_fwd(const attn_params* p, const void* q, const void* k, const void* v, void* o,
                     float* lse, void* workspace, size_t workspace_bytes, void* stream_) {
  (void)workspace;
  (void)workspace_bytes;
  attn_status st = attn_check_params(p, 0);
  if (st != ATTN_OK) return st;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (p->batch == 0 || p->seqlen_q == 0) return ATTN_OK;
  if (!o || !lse) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(o) || (reinterpret_cast<uintptr_t>(lse) & 3u)) return ATTN_ERR_MISALIGNED;
  if (p->seqlen_k == 0) {
    const long long n_o = (long long)p->batch * p->seqlen_q * p->nheads * p->headdim;
    const long long n_l = (long long)p->batch * p->nheads * p->seqlen_q;
    fill_empty_fwd<<<fill_blocks(n_o), 256, 0, stream>>>(static_cast<uint16_t*>(o), n_o, lse, n_l);
    return finish(stream);
  }
  if (!q || !k || !v) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v)) return ATTN_ERR_MISALIGNED;
  return dispatch_fwd(p, q, k, v, o, lse, stream, Packed());
}

size_t attn_bwd_workspace_size(const attn_params* p) {
  if (attn_check_params(p, 1) != ATTN_OK) return 0;
  return bwd_workspace_layout(p->batch, p->nheads, p->seqlen_q, p->headdim).total;
}

attn_status attn_bwd_prepare(const attn_params* p, const void* o, const float* lse,
                             const void* dout, void* workspace, size_t workspace_bytes,
                             void* stream_) {
  bool empty = false;
  attn_status st = bwd_common_checks(p, workspace, workspace_bytes, &empty);
  if (st != ATTN_OK || empty) return st;
  if (!o || !lse || !dout) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(o) || !aligned16(dout) || (reinterpret_cast<uintptr_t>(lse) & 3u))
    return ATTN_ERR_MISALIGNED;
  return launch_bwd_prepare(p, o, lse, dout, workspace, reinterpret_cast<cudaStream_t>(stream_));
}

attn_status attn_bwd_accumulate(const attn_params* p, const void* q, const void* k, const void* v,
                                const void* dout, void* dk, void* dv, void* workspace,
                                size_t workspace_bytes, void* stream_) {
  bool empty = false;
  attn_status st = bwd_common_checks(p, workspace, workspace_bytes, &empty);
  if (st != ATTN_OK || empty) return st;
  if (!q || !k || !v || !dout || !dk || !dv) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dout) || !aligned16(dk) ||
      !aligned16(dv))
    return ATTN_ERR_MISALIGNED;
  return dispatch_bwd_main(p, q, k, v, dout, dk, dv, workspace,
                           reinterpret_cast<cudaStream_t>(stream_), Packed());
}

attn_status attn_bwd_accumulate_f32(const attn_params* p, const void* q, const void* k,
                                    const void* v, const void* dout, float* dk_acc, float* dv_acc,
                                    void* workspace, size_t workspace_bytes, void* stream_) {
  bool empty = false;
  attn_status st = bwd_common_checks(p, workspace, workspace_bytes, &empty);
  if (st != ATTN_OK || empty) return st;
  if (drop_threshold(p->dropout_p) != 0) return ATTN_ERR_INVALID_ARG;
  if (!q || !k || !v || !dout || !dk_acc || !dv_acc) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dout) || !aligned16(dk_acc) ||
      !aligned16(dv_acc))
    return ATTN_ERR_MISALIGNED;
  return dispatch_bwd_main(p, q, k, v, dout, dk_acc, dv_acc, workspace,
                           reinterpret_cast<cudaStream_t>(stream_), Packed(), true);
}

attn_status attn_f32_to_16(const float* src, void* dst, long long n, int dtype, void* stream_) {
  if (n < 0 || (dtype != ATTN_BF16 && dtype != ATTN_FP16)) return ATTN_ERR_INVALID_ARG;
  if (n == 0) return ATTN_OK;
  if (!src || !dst || (n & 3)) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(src) || (reinterpret_cast<uintptr_t>(dst) & 7u)) return ATTN_ERR_MISALIGNED;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  BwdParams bp;
  std::memset(&bp, 0, sizeof(bp));  // cu_q == nullptr: a plain element-wise conversion
  if (dtype == ATTN_FP16)
    bwd_convert<true><<<2368, 256, 0, stream>>>(src, static_cast<uint16_t*>(dst), n / 4, 1.f, bp);
  else
    bwd_convert<false><<<2368, 256, 0, stream>>>(src, static_cast<uint16_t*>(dst), n / 4, 1.f, bp);
  return finish(stream);
}

attn_status attn_bwd_finalize(const attn_params* p, void* dq, void* workspace,
                              size_t workspace_bytes, void* stream_) {
  bool empty = false;
  attn_status st = bwd_common_checks(p, workspace, workspace_bytes, &empty);
  if (st != ATTN_OK || empty) return st;
  if (!dq) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(dq)) return ATTN_ERR_MISALIGNED;
  return launch_bwd_finalize(p, dq, workspace, reinterpret_cast<cudaStream_t>(stream_));
}

attn_status attn_bwd(const attn_params* p, const void* q, const void* k, const void* v,
                     const void* o, const float* lse, const void* dout, void* dq, void* dk,
                     void* dv, void* workspace, size_t workspace_bytes, void* stream_) {
  attn_status st = attn_check_params(p, 1);
  if (st != ATTN_OK) return st;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (p->batch == 0) return ATTN_OK;
  const long long n_q = (long long)p->batch * p->seqlen_q * p->nheads * p->headdim;
  const long long n_k = (long long)p->batch * p->seqlen_k * p->nheads_kv * p->headdim;
  if (p->seqlen_q == 0 || p->seqlen_k == 0) {
    // Nothing to attend: every gradient is zero.
    if ((n_q && !dq) || (n_k && (!dk || !dv))) return ATTN_ERR_INVALID_ARG;
    if ((n_q && !aligned16(dq)) || (n_k && (!aligned16(dk) || !aligned16(dv))))
      return ATTN_ERR_MISALIGNED;
    if (n_q) fill_zero_u16<<<fill_blocks(n_q), 256, 0, stream>>>(static_cast<uint16_t*>(dq), n_q);
    if (n_k) {
      fill_zero_u16<<<fill_blocks(n_k), 256, 0, stream>>>(static_cast<uint16_t*>(dk), n_k);
      fill_zero_u16<<<fill_blocks(n_k), 256, 0, stream>>>(static_cast<uint16_t*>(dv), n_k);
    }
    return finish(stream);
  }
  if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u))
    return ATTN_ERR_MISALIGNED;
  st = attn_bwd_prepare(p, o, lse, dout, workspace, workspace_bytes, stream_);
  if (st != ATTN_OK) return st;
  st = attn_bwd_accumulate(p, q, k, v, dout, dk, dv, workspace, workspace_bytes, stream_);
  if (st != ATTN_OK) return st;
  return attn_bwd_finalize(p, dq, workspace, workspace_bytes, stream_);
}

attn_status attn_bwd_noalloc(const attn_params* p, const void* q, const void* k, const void* v,
                             const void* o, const float* lse, const void* dout, void* dq, void* dk,
                             void* dv, void* stream_) {
  attn_status st = attn_check_params(p, 1);
  if (st != ATTN_OK) return st;
  if (p->batch == 0 || p->seqlen_q == 0 || p->seqlen_k == 0)  // no scratch needed
    return attn_bwd(p, q, k, v, o, lse, dout, dq, dk, dv, nullptr, 0, stream_);
  if (attn_bwd_workspace_size(p) > (size_t)ATTN_NOALLOC_SCRATCH_BYTES)
    return ATTN_ERR_WORKSPACE_TOO_SMALL;
  void* scratch = noalloc_scratch_address();
  if (!scratch) return ATTN_ERR_CUDA;
  // attn_bwd's first stage rewrites the row statistics and zeroes the dQ
  // accumulator, so the previous call's contents never leak into this one.
  return attn_bwd(p, q, k, v, o, lse, dout, dq, dk, dv, scratch, ATTN_NOALLOC_SCRATCH_BYTES,
                  stream_);
}

attn_status attn_get_device_status(void* stream_, int* code) {
  if (!code) return ATTN_ERR_INVALID_ARG;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  unsigned int host = 0, zero = 0;
  if (cudaMemcpyFromSymbolAsync(&host, g_attn_status, sizeof(host), 0, cudaMemcpyDeviceToHost,
                                stream) != cudaSuccess)
    return ATTN_ERR_CUDA;
  if (cudaMemcpyToSymbolAsync(g_attn_status, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice,
                              stream) != cudaSuccess)
    return ATTN_ERR_CUDA;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return ATTN_ERR_CUDA;
  *code = static_cast<int>(host);
  return ATTN_OK;
}

attn_status attn_check_varlen_params(const attn_varlen_params* v, int pass) {
  if (!v) return ATTN_ERR_INVALID_ARG;
  if (v->total_q < 0 || v->total_k < 0 || v->max_seqlen_q < 0 || v->max_seqlen_k < 0)
    return ATTN_ERR_INVALID_ARG;
  const attn_params p = packed_view(v);
  return attn_check_params(&p, pass);
}

size_t attn_bwd_varlen_workspace_size(const attn_varlen_params* v) {
  if (attn_check_varlen_params(v, 1) != ATTN_OK) return 0;
  return bwd_workspace_layout_packed(v->total_q, v->batch, v->nheads, v->headdim).total;
}

attn_status attn_fwd_varlen(const attn_varlen_params* v, const int32_t* cu_seqlens_q,
                            const int32_t* cu_seqlens_k, const void* q, const void* k,
                            const void* vv, void* o, float* lse, void* workspace,
                            size_t workspace_bytes, void* stream_) {
  (void)workspace;
  (void)workspace_bytes;
  attn_status st = attn_check_varlen_params(v, 0);
  if (st != ATTN_OK) return st;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (v->batch == 0 || v->total_q == 0 || v->max_seqlen_q == 0) return ATTN_OK;
  if (!o || !lse || !cu_seqlens_q || !cu_seqlens_k) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(o) || (reinterpret_cast<uintptr_t>(lse) & 3u) ||
      (reinterpret_cast<uintptr_t>(cu_seqlens_q) & 3u) ||
      (reinterpret_cast<uintptr_t>(cu_seqlens_k) & 3u))
    return ATTN_ERR_MISALIGNED;
  if (v->total_k == 0 || v->max_seqlen_k == 0) {
    const long long n_o = (long long)v->total_q * v->nheads * v->headdim;
    const long long n_l = (long long)v->nheads * v->total_q;
    fill_empty_fwd<<<fill_blocks(n_o), 256, 0, stream>>>(static_cast<uint16_t*>(o), n_o, lse, n_l);
    return finish(stream);
  }
  if (!q || !k || !vv) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(vv)) return ATTN_ERR_MISALIGNED;
  const attn_params p = packed_view(v);
  Packed pk;
  pk.cu_q = cu_seqlens_q;
  pk.cu_k = cu_seqlens_k;
  pk.total_q = v->total_q;
  pk.total_k = v->total_k;
  return dispatch_fwd(&p, q, k, vv, o, lse, stream, pk);
}

attn_status attn_bwd_varlen(const attn_varlen_params* v, const int32_t* cu_seqlens_q,
                            const int32_t* cu_seqlens_k, const void* q, const void* k,
                            const void* vv, const void* o, const float* lse, const void* dout,
                            void* dq, void* dk, void* dv, void* workspace,
                            size_t workspace_bytes, void* stream_) {
  attn_status st = attn_check_varlen_params(v, 1);
  if (st != ATTN_OK) return st;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (v->batch == 0) return ATTN_OK;
  const long long n_q = (long long)v->total_q * v->nheads * v->headdim;
  const long long n_k = (long long)v->total_k * v->nheads_kv * v->headdim;
  if ((n_q && !dq) || (n_k && (!dk || !dv))) return ATTN_ERR_INVALID_ARG;
  if ((n_q && !aligned16(dq)) || (n_k && (!aligned16(dk) || !aligned16(dv))))
    return ATTN_ERR_MISALIGNED;
  if (n_q == 0 || n_k == 0 || v->max_seqlen_q == 0 || v->max_seqlen_k == 0) {
    // Nothing to attend: every gradient is zero.
    if (n_q) fill_zero_u16<<<fill_blocks(n_q), 256, 0, stream>>>(static_cast<uint16_t*>(dq), n_q);
    if (n_k) {
      fill_zero_u16<<<fill_blocks(n_k), 256, 0, stream>>>(static_cast<uint16_t*>(dk), n_k);
      fill_zero_u16<<<fill_blocks(n_k), 256, 0, stream>>>(static_cast<uint16_t*>(dv), n_k);
    }
    return finish(stream);
  }
  if (!q || !k || !vv || !o || !lse || !dout || !cu_seqlens_q || !cu_seqlens_k)
    return ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(vv) || !aligned16(o) || !aligned16(dout) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u) ||
      (reinterpret_cast<uintptr_t>(cu_seqlens_q) & 3u) ||
      (reinterpret_cast<uintptr_t>(cu_seqlens_k) & 3u))
    return ATTN_ERR_MISALIGNED;
  if (!workspace || workspace_bytes < attn_bwd_varlen_workspace_size(v))
    return ATTN_ERR_WORKSPACE_TOO_SMALL;
  if (reinterpret_cast<uintptr_t>(workspace) & 255u) return ATTN_ERR_MISALIGNED;
  const attn_params p = packed_view(v);
  Packed pk;
  pk.cu_q = cu_seqlens_q;
  pk.cu_k = cu_seqlens_k;
  pk.total_q = v->total_q;
  pk.total_k = v->total_k;
  st = launch_bwd_prepare(&p, o, lse, dout, workspace, stream, pk);
  if (st != ATTN_OK) return st;
  st = dispatch_bwd_main(&p, q, k, vv, dout, dk, dv, workspace, stream, pk);
  if (st != ATTN_OK) return st;
  return launch_bwd_finalize(&p, dq, workspace, stream, pk);
}

attn_status attn_merge(const attn_merge_params* p, const void* o_parts, const float* lse_parts,
                       void* o, float* lse, void* stream_) {
  if (!p || p->splits < 1 || p->splits > 65535 || p->batch < 0 || p->seqlen_q < 0 ||
      p->nheads < 1)
    return ATTN_ERR_INVALID_ARG;
  if (p->headdim != 64 && p->headdim != 128 && p->headdim != 256)
    return ATTN_ERR_UNSUPPORTED_HEADDIM;
  if (p->dtype != ATTN_BF16 && p->dtype != ATTN_FP16) return ATTN_ERR_UNSUPPORTED_DTYPE;
  const long long rows = (long long)p->batch * p->seqlen_q * p->nheads;
  if (rows == 0) return ATTN_OK;
  if (!o_parts || !lse_parts || !o || !lse) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(o_parts) || !aligned16(o) || (reinterpret_cast<uintptr_t>(lse_parts) & 3u) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u))
    return ATTN_ERR_MISALIGNED;
  MergeParams mp;
  mp.o_parts = static_cast<const uint16_t*>(o_parts);
  mp.lse_parts = lse_parts;
  mp.o = static_cast<uint16_t*>(o);
  mp.lse = lse;
  mp.splits = p->splits;
  mp.nq = p->seqlen_q;
  mp.nheads = p->nheads;
  mp.headdim = p->headdim;
  mp.rows = rows;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  const long long rows_per_block = 8LL * (32 / (p->headdim / 8));
  long long blocks = (rows + rows_per_block - 1) / rows_per_block;
  if (blocks > 4736) blocks = 4736;  // 32 x 148 SMs, grid-stride beyond
  if (p->dtype == ATTN_FP16)
    attn_merge_kernel<true><<<(unsigned)blocks, 256, 0, stream>>>(mp);
  else
    attn_merge_kernel<false><<<(unsigned)blocks, 256, 0, stream>>>(mp);
  return finish(stream);
}

attn_status attn_selftest_bounded_wait(unsigned int wait_limit_us, int* result, void* stream_) {
  if (wait_limit_us == 0 || wait_limit_us > 1000000u) return ATTN_ERR_INVALID_ARG;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  selftest_bounded_wait_kernel<<<1, 64, 0, stream>>>(1000ull * wait_limit_us, result);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // extern "C"
