// fa_api.cu -- the C ABI (include/fa.h): argument validation, TMA tensor-map
// encoding, per-device set-up and kernel launches on the caller's stream.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <mutex>

#include "../../include/fa.h"
#include "bwd_fused.cuh"
#include "bwd_kernels.cuh"
#include "decode_kernel.cuh"
#include "fp8_quant.cuh"
#include "fwd_kernel.cuh"

namespace {

__device__ int g_error_word;   // bounded-wait timeouts are recorded here

constexpr int kMaxDevices = 64;
constexpr unsigned long long kDefaultTimeoutNs = 2000000000ull;

// ----------------------------------------------------------- profiling --
// Event pairs recorded around each launch while profiling is on.
// forward, D pre-pass, dK/dV, dQ, decode, merge, FP8 quantise, FP8 forward,
// fused backward kernel, fused backward's dQ conversion
constexpr int kProfKinds = 10;
constexpr int kProfCap = 1024;
constexpr int kClockCtas = 4096;   // CTA timing entries of the profiled forward launch
struct Profiler {
    bool created = false;
    bool on = false;
    int device = -1;
    cudaEvent_t ev[kProfKinds][kProfCap][2];
    int n[kProfKinds] = {};
    unsigned long long* cta_clock = nullptr;   // device: 1 + 2 * kClockCtas entries
};
thread_local Profiler g_prof;

// Records the "before" event of a launch of `kind`; returns the slot or -1.
int prof_start(int kind, cudaStream_t stream) {
    Profiler& P = g_prof;
    if (!P.on || P.n[kind] >= kProfCap) return -1;
    const int slot = P.n[kind]++;
    cudaEventRecord(P.ev[kind][slot][0], stream);
    return slot;
}
void prof_stop(int kind, int slot, cudaStream_t stream) {
    if (slot >= 0) cudaEventRecord(g_prof.ev[kind][slot][1], stream);
}

int g_fault_mode = 0;
unsigned long long g_fault_timeout_ns = 0;

struct DeviceState {
    bool ready = false;
    int num_sms = 0;
    int* error_word = nullptr;
};
DeviceState g_dev[kMaxDevices];
std::mutex g_mutex;

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

// The warp-specialised kernels (forward, dK/dV, dQ, fused backward) hand
// registers between their warpgroups with setmaxnreg; the shares add up to
// 168 per thread over their 384 threads, which must not exceed what a kernel
// was launched with, or the increase would wait forever.  A build whose
// kernels came out with fewer registers is refused at set-up.
template <typename K>
bool regs_pool_ok(K kernel) {
    cudaFuncAttributes a;
    return cudaFuncGetAttributes(&a, reinterpret_cast<const void*>(kernel)) == cudaSuccess &&
           a.numRegs >= 168;
}

template <typename K>
cudaError_t allow_smem(K kernel, int bytes) {
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

template <int D>
cudaError_t decode_set_smem_limits_d() {
    const int b = fa::DecCfg<D>::SMEM_BYTES;
    cudaError_t e = allow_smem(fa::decode_kernel<D, 1>, b);
    if (e == cudaSuccess) e = allow_smem(fa::decode_kernel<D, 2>, b);
    if (e == cudaSuccess) e = allow_smem(fa::decode_kernel<D, 4>, b);
    if (e == cudaSuccess) e = allow_smem(fa::decode_kernel<D, 8>, b);
    if (e == cudaSuccess) e = allow_smem(fa::decode_kernel<D, 16>, b);
    return e;
}

cudaError_t decode_set_smem_limits() {
    cudaError_t e = decode_set_smem_limits_d<64>();
    return e == cudaSuccess ? decode_set_smem_limits_d<128>() : e;
}

// Per-device one-time set-up: SM count, the device address of the error word,
// the driver's tensor-map encoder and the kernels' shared-memory limits.
int device_setup(DeviceState** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mutex);
    DeviceState& st = g_dev[dev];
    if (!st.ready) {
        if (cudaDeviceGetAttribute(&st.num_sms, cudaDevAttrMultiProcessorCount, dev) !=
            cudaSuccess)
            return FA_ERR_CUDA;
        if (cudaGetSymbolAddress(reinterpret_cast<void**>(&st.error_word), g_error_word) !=
            cudaSuccess)
            return FA_ERR_CUDA;
        if (!g_encode) {
            void* fn = nullptr;
            cudaDriverEntryPointQueryResult q;
            if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
                    cudaSuccess ||
                q != cudaDriverEntryPointSuccess || !fn)
                return FA_ERR_CUDA;
            g_encode = reinterpret_cast<EncodeTiledFn>(fn);
        }
        if (allow_smem(fa::fwd_kernel<64>, fa::FwdCfg<64>::SMEM_BYTES) != cudaSuccess ||
            allow_smem(fa::fwd_kernel<128>, fa::FwdCfg<128>::SMEM_BYTES) != cudaSuccess ||
            decode_set_smem_limits() != cudaSuccess ||
            allow_smem(fa::fwd_kernel<128, true>, fa::FwdCfg<128, true>::SMEM_BYTES) != cudaSuccess ||
            allow_smem(fa::fwd_kernel<64, false, true>, fa::FwdCfg<64>::SMEM_BYTES) != cudaSuccess ||
            allow_smem(fa::fwd_kernel<128, false, true>, fa::FwdCfg<128>::SMEM_BYTES) != cudaSuccess ||
            allow_smem(fa::fwd_kernel<64, false, false, true>, fa::FwdCfg<64>::SMEM_BYTES) != cudaSuccess ||
            allow_smem(fa::fwd_kernel<128, false, false, true>, fa::FwdCfg<128>::SMEM_BYTES) != cudaSuccess ||
            allow_smem(fa::quantize_fp8_kernel<true, false>, fa::QuantCfg::SMEM_BYTES) != cudaSuccess ||
            allow_smem(fa::quantize_fp8_kernel<false, false>, fa::QuantCfg::SMEM_BYTES) != cudaSuccess ||
            allow_smem(fa::quantize_fp8_kernel<false, true>, fa::QuantCfg::SMEM_BYTES) != cudaSuccess ||
            fa::bwd_set_smem_limits() != cudaSuccess || fa::fused_set_smem_limit() != cudaSuccess)
            return FA_ERR_CUDA;
        if (!regs_pool_ok(fa::fwd_kernel<64>) || !regs_pool_ok(fa::fwd_kernel<128>) ||
            !regs_pool_ok(fa::fwd_kernel<128, true>) || !regs_pool_ok(fa::fwd_kernel<64, false, true>) ||
            !regs_pool_ok(fa::fwd_kernel<128, false, true>) ||
            !regs_pool_ok(fa::fwd_kernel<64, false, false, true>) ||
            !regs_pool_ok(fa::fwd_kernel<128, false, false, true>) || !regs_pool_ok(fa::dkdv_kernel<64>) ||
            !regs_pool_ok(fa::dkdv_kernel<128>) || !regs_pool_ok(fa::dq_kernel<64>) ||
            !regs_pool_ok(fa::dq_kernel<128>) || !regs_pool_ok(fa::dkdvq_kernel))
            return FA_ERR_CUDA;
        st.ready = true;
    }
    *out = &st;
    return FA_OK;
}

// Tensor map over a token-major [rows, H, d] bf16 tensor; boxes of
// 64 channels x 1 head x box_rows tokens, 128-byte swizzle, zero fill outside.
int make_map(CUtensorMap* map, const void* ptr, int64_t rows, int H, int d, int box_rows) {
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(H),
                          static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2,
                             static_cast<cuuint64_t>(H) * static_cast<cuuint64_t>(d) * 2};
    cuuint32_t box[3] = {64, 1, static_cast<cuuint32_t>(box_rows)};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? FA_OK : FA_ERR_CUDA;
}

// Tensor map over a padded cache [B, rows, H, d] bf16 tensor, coordinates
// (channel, head, row, sequence); boxes of 64 channels x 1 head x box_rows
// rows x 1 sequence (the same shared-memory layout as make_map's boxes),
// 128-byte swizzle, zero fill outside -- so a box that starts at a negative
// row never reads the sequence before it.
int make_map_cache(CUtensorMap* map, const void* ptr, int B, int rows, int H, int d, int box_rows) {
    const cuuint64_t row_bytes = static_cast<cuuint64_t>(H) * static_cast<cuuint64_t>(d) * 2;
    cuuint64_t dims[4] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(H),
                          static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(B)};
    cuuint64_t strides[3] = {static_cast<cuuint64_t>(d) * 2, row_bytes,
                             row_bytes * static_cast<cuuint64_t>(rows)};
    cuuint32_t box[4] = {64, 1, static_cast<cuuint32_t>(box_rows), 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? FA_OK : FA_ERR_CUDA;
}

bool misaligned(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) != 0; }

// FP8 operands: e4m3 codes [rows, H, 128] (3-D, boxes of 128 channels x 1 head x
// 128 rows) and transposed V codes [B*H*128, Np] (2-D, boxes of 128 keys x 128
// channel rows); 128-byte swizzle, zero fill outside.
int make_map_u8_3d(CUtensorMap* map, const void* ptr, int64_t rows, int H) {
    cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[2] = {128, static_cast<cuuint64_t>(H) * 128};
    cuuint32_t box[3] = {128, 1, 128};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(ptr), dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? FA_OK : FA_ERR_CUDA;
}

int make_map_u8_2d(CUtensorMap* map, const void* ptr, int64_t rows, int64_t cols) {
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols)};
    cuuint32_t box[2] = {128, 128};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(ptr), dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? FA_OK : FA_ERR_CUDA;
}

int64_t fp8_vt_pitch(int N) { return (static_cast<int64_t>(N) + 15) / 16 * 16; }

struct Common {
    fa::Geometry g;
    int64_t rows;      // token rows of the [rows, H, d] buffers
};

int validate_common(int B, int H, int N, int d, float scale, int causal, int window,
                    const int* cu_seqlens, Common* c) {
    if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED_D;
    if (B < 0 || H <= 0 || N < 0) return FA_ERR_BAD_SHAPE;
    if (!(scale > 0.f) || !std::isfinite(scale)) return FA_ERR_BAD_SCALE;
    if (window > 0 && !causal) return FA_ERR_BAD_MASK;
    if (cu_seqlens && B > fa::kMaxVarlenSeqs) return FA_ERR_BAD_SHAPE;
    if (cu_seqlens && (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u)) return FA_ERR_MISALIGNED;
    const int64_t rows = cu_seqlens ? static_cast<int64_t>(N) : static_cast<int64_t>(B) * N;
    if (rows > (int64_t{1} << 31) - 1) return FA_ERR_BAD_SHAPE;
    if (rows * H * d > (int64_t{1} << 40)) return FA_ERR_BAD_SHAPE;
    c->rows = rows;
    c->g.B = B;
    c->g.H = H;
    c->g.N = cu_seqlens ? 0 : N;
    c->g.T = static_cast<int>(rows);
    c->g.cu_seqlens = cu_seqlens;
    c->g.causal = causal ? 1 : 0;
    c->g.window = window > 0 ? window : 0;
    // self-attention: the key/value sequences are the query sequences
    c->g.Nk = c->g.N;
    c->g.Tk = c->g.T;
    c->g.cu_seqlens_k = cu_seqlens;
    return FA_OK;
}

template <int D, bool kSingles = false>
int launch_fwd(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
               const fa::FwdParams& p, int grid, cudaStream_t stream) {
    fa::fwd_kernel<D, false, false, kSingles><<<grid, fa::FwdCfg<D>::THREADS, fa::FwdCfg<D>::SMEM_BYTES,
                                                 stream>>>(mq, mk, mv, p);
    return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

// The padded-cache instantiation: 4-D K/V maps (make_map_cache), one block
// per work unit, optional split along the keys (p.nsplit).
template <int D>
int launch_fwd_cache(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                     const fa::FwdParams& p, int grid, cudaStream_t stream) {
    fa::fwd_kernel<D, false, true><<<grid, fa::FwdCfg<D>::THREADS, fa::FwdCfg<D>::SMEM_BYTES,
                                      stream>>>(mq, mk, mv, p);
    return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

// ------------------------------------------------------ decode / split-KV --
// Split count for a decode call: each split gets at least 4 key tiles (256
// keys); among the counts up to that limit, the smallest whose CTAs fill the
// GPU's slots (two CTAs per SM) to at least 90 % of whole waves, else the
// best-filling one.
int decode_splits(int B, int H, int Nk, int num_sms) {
    const int64_t items = static_cast<int64_t>(B) * H;
    const int tiles = (Nk + 63) / 64;
    const int max_ns = std::max(1, std::min(fa::kDecMaxSplits, tiles / 4));
    const int64_t slots = 2 * static_cast<int64_t>(num_sms);
    int best = 1;
    double best_fill = -1.0;
    for (int ns = 1; ns <= max_ns; ++ns) {
        const int64_t ctas = items * ns;
        const int64_t waves = (ctas + slots - 1) / slots;
        const double fill = static_cast<double>(ctas) / static_cast<double>(waves * slots);
        if (fill >= 0.9) return ns;
        if (fill > best_fill + 1e-9) {
            best_fill = fill;
            best = ns;
        }
    }
    return best;
}

// Split count for a prefill chunk (more than 16 queries) on the tensor-core
// forward, whose work items are blocks of 256 queries: split only when there
// are fewer blocks than SMs, into as many ranges as fill them, each keeping at
// least 8 key tiles of 128.  (With enough blocks, splitting measured slower:
// the extra Q loads and fp32 partial outputs cost more than the better
// balance of the last wave gains.)
int prefill_splits(int B, int H, int Nq, int Nk, int num_sms) {
    const int64_t items = static_cast<int64_t>(B) * H * ((Nq + 255) / 256);
    if (items >= num_sms) return 1;
    const int tiles = (Nk + 127) / 128;
    const int64_t want = (num_sms + items - 1) / items;
    return static_cast<int>(std::max<int64_t>(1, std::min<int64_t>({want, fa::kDecMaxSplits, tiles / 8})));
}

int kvcache_splits(int B, int H, int Nq, int Nk, int num_sms) {
    return Nq <= fa::kDecMaxQ ? decode_splits(B, H, Nk, num_sms)
                              : prefill_splits(B, H, Nq, Nk, num_sms);
}

size_t decode_workspace_bytes(int B, int H, int Nq, int d, int ns) {
    if (ns <= 1) return 0;
    const size_t rows = static_cast<size_t>(B) * Nq;
    const size_t bytes = static_cast<size_t>(ns) * rows * H * (static_cast<size_t>(d) + 1) * 4;
    return (bytes + 255) & ~static_cast<size_t>(255);
}

template <int D>
int launch_decode(const CUtensorMap& mk, const CUtensorMap& mv, const fa::DecodeParams& p,
                  cudaStream_t stream) {
    const int grid = p.B * p.H * p.nsplit;
    constexpr int T = fa::DecCfg<D>::THREADS, S = fa::DecCfg<D>::SMEM_BYTES;
    const int slot = prof_start(4, stream);
    if (p.Nq <= 1)
        fa::decode_kernel<D, 1><<<grid, T, S, stream>>>(mk, mv, p);
    else if (p.Nq <= 2)
        fa::decode_kernel<D, 2><<<grid, T, S, stream>>>(mk, mv, p);
    else if (p.Nq <= 4)
        fa::decode_kernel<D, 4><<<grid, T, S, stream>>>(mk, mv, p);
    else if (p.Nq <= 8)
        fa::decode_kernel<D, 8><<<grid, T, S, stream>>>(mk, mv, p);
    else
        fa::decode_kernel<D, 16><<<grid, T, S, stream>>>(mk, mv, p);
    prof_stop(4, slot, stream);
    if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
    if (p.nsplit > 1) {
        const int64_t warps = static_cast<int64_t>(p.B) * p.Nq * p.H;
        const int blocks = static_cast<int>((warps + 7) / 8);
        const int slot2 = prof_start(5, stream);
        // programmatic dependent launch: the merge's CTAs are scheduled while
        // the split kernel's last wave runs and wait on the device for it
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(blocks);
        cfg.blockDim = dim3(256);
        cfg.dynamicSmemBytes = 0;
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        const cudaError_t e = cudaLaunchKernelEx(&cfg, fa::combine_kernel<D>, p.o_part, p.lse_part, p.o,
                                                 p.lse, p.B * p.Nq, p.H, p.Nq, p.nsplit);
        prof_stop(5, slot2, stream);
        if (e != cudaSuccess || cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
    }
    return FA_OK;
}

// ------------------------------------------------ allocation-free backward --
// Built-in scratch for fa_bwd_noalloc: the per-row statistics (two floats a
// row, padded to 128-row blocks) of one backward call.  In
// host code the symbol is only a host-side stand-in; kernels get the device
// address looked up once per device below.
static __device__ __align__(256) float2 g_noalloc_scratch[FA_NOALLOC_MAX_ROWS];

struct NoAllocState {
    bool ready = false;
    float2* scratch = nullptr;  // device address of g_noalloc_scratch on this device
};
NoAllocState g_noalloc[kMaxDevices];

// One-time, per-device lookup of the scratch array's device address (with
// that device current).
int noalloc_setup(float2** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mutex);
    NoAllocState& st = g_noalloc[dev];
    if (!st.ready) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr)
            return FA_ERR_CUDA;
        st.scratch = static_cast<float2*>(ptr);
        st.ready = true;
    }
    *out = st.scratch;
    return FA_OK;
}

}  // namespace

extern "C" {

int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N,
           int d, float scale, int causal, int window, const int* cu_seqlens,
           cudaStream_t stream) {
    return fa_fwd_kv(q, k, v, o, lse, B, H, N, N, d, scale, causal, window, cu_seqlens,
                     cu_seqlens, stream);
}

int fa_fwd_kv(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
              int Nq, int Nk, int d, float scale, int causal, int window,
              const int* cu_seqlens_q, const int* cu_seqlens_k, cudaStream_t stream) {
    if (!q || !o || !lse) return FA_ERR_NULLPTR;
    Common c;
    int rc = validate_common(B, H, Nq, d, scale, causal, window, cu_seqlens_q, &c);
    if (rc != FA_OK) return rc;
    if (Nk < 0 || (cu_seqlens_q == nullptr) != (cu_seqlens_k == nullptr)) return FA_ERR_BAD_SHAPE;
    if (cu_seqlens_k && (reinterpret_cast<uintptr_t>(cu_seqlens_k) & 3u)) return FA_ERR_MISALIGNED;
    const bool packed = cu_seqlens_q != nullptr;
    const int64_t rows_k = packed ? static_cast<int64_t>(Nk) : static_cast<int64_t>(B) * Nk;
    if (rows_k > (int64_t{1} << 31) - 1 || rows_k * H * d > (int64_t{1} << 40))
        return FA_ERR_BAD_SHAPE;
    if (rows_k > 0 && (!k || !v)) return FA_ERR_NULLPTR;   // k, v may be NULL without key rows
    c.g.Nk = packed ? 0 : Nk;
    c.g.Tk = static_cast<int>(rows_k);
    c.g.cu_seqlens_k = cu_seqlens_k;
    if (misaligned(q) || misaligned(k) || misaligned(v) || misaligned(o) || misaligned(lse))
        return FA_ERR_MISALIGNED;
    if (B == 0 || c.rows == 0) return FA_OK;
    DeviceState* st = nullptr;
    if ((rc = device_setup(&st)) != FA_OK) return rc;

    // Fixed length with at least twice as many keys as queries (a chunk of
    // queries after a cached prefix): the padded-cache instantiation, which
    // deals every query block as its own work unit, so that the CTAs running
    // at once share the K/V of few enough heads to stay in L2 (pairs of
    // blocks on one CTA spread them over twice as many).
    if (!packed && Nk > 0 && Nk >= 2 * static_cast<int64_t>(Nq)) {
        CUtensorMap mq, mk, mv;
        if (static_cast<int64_t>(Nk) * H * d * 2 >= (int64_t{1} << 40)) return FA_ERR_BAD_SHAPE;
        if (make_map(&mq, q, c.rows, H, d, 128) || make_map_cache(&mk, k, B, Nk, H, d, 128) ||
            make_map_cache(&mv, v, B, Nk, H, d, 128))
            return FA_ERR_CUDA;
        fa::FwdParams p;
        p.g = c.g;
        p.o = static_cast<__nv_bfloat16*>(o);
        p.lse = lse;
        p.scale_log2 = scale * 1.4426950408889634f;
        p.error_word = st->error_word;
        p.timeout_ns = g_fault_timeout_ns ? g_fault_timeout_ns : kDefaultTimeoutNs;
        p.fault_skip_v = g_fault_mode == 1 ? 1 : 0;
        p.nsplit = 1;
        p.kv.seqused_k = nullptr;
        p.kv.o_part = nullptr;
        p.kv.lse_part = nullptr;
        int grid = st->num_sms;
        const int64_t items = static_cast<int64_t>(B) * H * ((Nq + 255) / 256);
        if (items < grid) grid = static_cast<int>(items);
        const int slot = prof_start(0, stream);
        rc = d == 64 ? launch_fwd_cache<64>(mq, mk, mv, p, grid, stream)
                     : launch_fwd_cache<128>(mq, mk, mv, p, grid, stream);
        prof_stop(0, slot, stream);
        return rc;
    }

    // With no key rows at all every key tile is fully masked (each sequence
    // has nk = 0), but a tensor map cannot be empty: point the K/V maps at q,
    // whose tiles are then loaded, masked and contribute nothing.
    const void* kk = rows_k > 0 ? k : q;
    const void* vv = rows_k > 0 ? v : q;
    const int64_t map_rows_k = rows_k > 0 ? rows_k : c.rows;
    CUtensorMap mq, mk, mv;
    if (make_map(&mq, q, c.rows, H, d, 128) || make_map(&mk, kk, map_rows_k, H, d, 128) ||
        make_map(&mv, vv, map_rows_k, H, d, 128))
        return FA_ERR_CUDA;

    fa::FwdParams p;
    p.g = c.g;
    p.o = static_cast<__nv_bfloat16*>(o);
    p.lse = lse;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.error_word = st->error_word;
    p.timeout_ns = g_fault_timeout_ns ? g_fault_timeout_ns : kDefaultTimeoutNs;
    p.fault_skip_v = g_fault_mode == 1 ? 1 : 0;

    int grid = st->num_sms;
    if (!packed) {
        const int64_t items = static_cast<int64_t>(B) * H * ((Nq + 255) / 256);
        if (items < grid) grid = static_cast<int>(items);
    }
    // packed batches holding at least twice as many key rows as query rows
    // (chunks after cached prefixes): one block per work unit, as for the
    // fixed-length case above
    const bool singles = packed && Nk >= 2 * static_cast<int64_t>(Nq);
    const int slot = prof_start(0, stream);
    if (singles)
        rc = d == 64 ? launch_fwd<64, true>(mq, mk, mv, p, grid, stream)
                     : launch_fwd<128, true>(mq, mk, mv, p, grid, stream);
    else
        rc = d == 64 ? launch_fwd<64>(mq, mk, mv, p, grid, stream)
                     : launch_fwd<128>(mq, mk, mv, p, grid, stream);
    prof_stop(0, slot, stream);
    return rc;
}

int fa_fwd_kvcache_num_splits(int B, int H, int Nq, int Nk, int d) {
    (void)d;
    if (B <= 0 || H <= 0 || Nk <= 0 || Nq <= 0) return 1;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (sms <= 0) sms = 148;
    return kvcache_splits(B, H, Nq, Nk, sms);
}

size_t fa_fwd_kvcache_workspace_size(int B, int H, int Nq, int d, int num_splits) {
    if (B <= 0 || H <= 0 || Nq <= 0 || d <= 0) return 0;
    return decode_workspace_bytes(B, H, Nq, d, num_splits);
}

int fa_fwd_kvcache(const void* q, const void* k_cache, const void* v_cache, void* o, float* lse,
                   int B, int H, int Nq, int Nk, int d, float scale, int causal, int window,
                   const int* seqlens_k, int num_splits, void* workspace, size_t workspace_bytes,
                   cudaStream_t stream) {
    if (!q || !o || !lse) return FA_ERR_NULLPTR;
    if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED_D;
    if (B < 0 || H <= 0 || Nq < 0 || Nk < 0) return FA_ERR_BAD_SHAPE;
    if (num_splits < 0 || num_splits > fa::kDecMaxSplits) return FA_ERR_BAD_SHAPE;
    if (!(scale > 0.f) || !std::isfinite(scale)) return FA_ERR_BAD_SCALE;
    if (window > 0 && !causal) return FA_ERR_BAD_MASK;
    const int64_t rows_q = static_cast<int64_t>(B) * Nq;
    const int64_t rows_k = static_cast<int64_t>(B) * Nk;
    if (rows_k > (int64_t{1} << 31) - 1 || rows_k * H * d > (int64_t{1} << 40) ||
        rows_q * H * d > (int64_t{1} << 40) || static_cast<int64_t>(B) * H * fa::kDecMaxSplits > (int64_t{1} << 31) - 1)
        return FA_ERR_BAD_SHAPE;
    if (rows_k > 0 && (!k_cache || !v_cache)) return FA_ERR_NULLPTR;
    if (misaligned(q) || misaligned(k_cache) || misaligned(v_cache) || misaligned(o) ||
        misaligned(lse) || (reinterpret_cast<uintptr_t>(seqlens_k) & 3u))
        return FA_ERR_MISALIGNED;
    if (rows_q == 0) return FA_OK;
    auto check_ws = [&](int ns) {
        const size_t need = decode_workspace_bytes(B, H, Nq, d, ns);
        if (need == 0) return FA_OK;
        if (!workspace || workspace_bytes < need) return FA_ERR_WORKSPACE;
        return misaligned(workspace) ? FA_ERR_MISALIGNED : FA_OK;
    };
    int rc = num_splits > 0 ? check_ws(num_splits) : FA_OK;
    if (rc != FA_OK) return rc;
    DeviceState* st = nullptr;
    if ((rc = device_setup(&st)) != FA_OK) return rc;
    const int ns = num_splits > 0 ? num_splits : kvcache_splits(B, H, Nq, Nk, st->num_sms);
    if ((rc = check_ws(ns)) != FA_OK) return rc;
    if (Nq > fa::kDecMaxQ) {
        // a prefill chunk: the tensor-core forward, split along the keys when ns > 1
        if (rows_q > (int64_t{1} << 31) - 1) return FA_ERR_BAD_SHAPE;
        // with no cache rows at all the maps are pointed at q: every key tile is
        // then read at rows [-128, 0), outside the map, so nothing of q is read
        const void* kk = rows_k > 0 ? k_cache : q;
        const void* vv = rows_k > 0 ? v_cache : q;
        const int map_rows_k = rows_k > 0 ? Nk : Nq;
        if (static_cast<int64_t>(map_rows_k) * H * d * 2 >= (int64_t{1} << 40)) return FA_ERR_BAD_SHAPE;
        CUtensorMap mq, mk, mv;
        if (make_map(&mq, q, rows_q, H, d, 128) || make_map_cache(&mk, kk, B, map_rows_k, H, d, 128) ||
            make_map_cache(&mv, vv, B, map_rows_k, H, d, 128))
            return FA_ERR_CUDA;
        fa::FwdParams p;
        p.g.B = B;
        p.g.H = H;
        p.g.N = Nq;
        p.g.T = static_cast<int>(rows_q);
        p.g.cu_seqlens = nullptr;
        p.g.causal = causal ? 1 : 0;
        p.g.window = window > 0 ? window : 0;
        p.g.Nk = Nk;
        p.g.Tk = static_cast<int>(rows_k);
        p.g.cu_seqlens_k = nullptr;
        p.o = static_cast<__nv_bfloat16*>(o);
        p.lse = lse;
        p.scale_log2 = scale * 1.4426950408889634f;
        p.error_word = st->error_word;
        p.timeout_ns = g_fault_timeout_ns ? g_fault_timeout_ns : kDefaultTimeoutNs;
        p.fault_skip_v = 0;
        p.nsplit = ns;
        p.kv.seqused_k = seqlens_k;
        p.kv.o_part = ns > 1 ? static_cast<float*>(workspace) : nullptr;
        p.kv.lse_part = ns > 1 ? static_cast<float*>(workspace) + static_cast<size_t>(ns) * rows_q * H * d
                               : nullptr;
        int grid = st->num_sms;
        const int64_t items = static_cast<int64_t>(B) * H * ns * ((Nq + 255) / 256);
        if (items < grid) grid = static_cast<int>(items);
        const int slot = prof_start(0, stream);
        rc = d == 64 ? launch_fwd_cache<64>(mq, mk, mv, p, grid, stream)
                     : launch_fwd_cache<128>(mq, mk, mv, p, grid, stream);
        prof_stop(0, slot, stream);
        if (rc != FA_OK || ns == 1) return rc;
        const int64_t warps = rows_q * H;
        const int slot2 = prof_start(5, stream);
        if (d == 64)
            fa::combine_kernel<64><<<static_cast<int>((warps + 7) / 8), 256, 0, stream>>>(
                p.kv.o_part, p.kv.lse_part, p.o, lse, static_cast<int>(rows_q), H, Nq, ns);
        else
            fa::combine_kernel<128><<<static_cast<int>((warps + 7) / 8), 256, 0, stream>>>(
                p.kv.o_part, p.kv.lse_part, p.o, lse, static_cast<int>(rows_q), H, Nq, ns);
        prof_stop(5, slot2, stream);
        return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
    }
    // With no cache rows every split is empty and no tile is loaded; the maps
    // still need a valid base, so they are pointed at q.
    const void* kk = rows_k > 0 ? k_cache : q;
    const void* vv = rows_k > 0 ? v_cache : q;
    const int64_t map_rows = rows_k > 0 ? rows_k : rows_q;
    CUtensorMap mk, mv;
    if (make_map(&mk, kk, map_rows, H, d, 64) || make_map(&mv, vv, map_rows, H, d, 64))
        return FA_ERR_CUDA;

    fa::DecodeParams p;
    p.q = static_cast<const __nv_bfloat16*>(q);
    p.o = static_cast<__nv_bfloat16*>(o);
    p.lse = lse;
    p.o_part = ns > 1 ? static_cast<float*>(workspace) : nullptr;
    p.lse_part = ns > 1 ? static_cast<float*>(workspace) + static_cast<size_t>(ns) * rows_q * H * d
                        : nullptr;
    p.seqlens_k = seqlens_k;
    p.B = B;
    p.H = H;
    p.Nq = Nq;
    p.Nk = Nk;
    p.causal = causal ? 1 : 0;
    p.window = window > 0 ? window : 0;
    p.nsplit = ns;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.error_word = st->error_word;
    p.timeout_ns = g_fault_timeout_ns ? g_fault_timeout_ns : kDefaultTimeoutNs;
    p.fault_skip = g_fault_mode == 2 ? 1 : 0;
    return d == 64 ? launch_decode<64>(mk, mv, p, stream) : launch_decode<128>(mk, mv, p, stream);
}

size_t fa_fp8_vt_bytes(int B, int H, int N, int d) {
    if (B <= 0 || H <= 0 || N <= 0 || d != 128) return 0;
    return static_cast<size_t>(B) * H * d * static_cast<size_t>(fp8_vt_pitch(N));
}

int fa_quantize_fp8(const void* x, void* out, float* scales, int B, int N, int H, int d,
                    int transpose, const float* signs, cudaStream_t stream) {
    if (!x || !out || !scales) return FA_ERR_NULLPTR;
    if (d != 128) return FA_ERR_UNSUPPORTED_D;
    if (B < 0 || N < 0 || H <= 0) return FA_ERR_BAD_SHAPE;
    if (transpose && signs) return FA_ERR_BAD_SHAPE;     // the rotation is for Q and K only
    const int64_t rows = static_cast<int64_t>(B) * N;
    const int64_t nb = (static_cast<int64_t>(N) + 127) / 128;
    if (rows * H * d > (int64_t{1} << 40) || static_cast<int64_t>(B) * H * nb > (int64_t{1} << 31) - 1)
        return FA_ERR_BAD_SHAPE;
    if (misaligned(x) || misaligned(out) || (reinterpret_cast<uintptr_t>(scales) & 3u) ||
        (reinterpret_cast<uintptr_t>(signs) & 3u))
        return FA_ERR_MISALIGNED;
    if (rows == 0) return FA_OK;
    DeviceState* st = nullptr;
    int rc = device_setup(&st);
    if (rc != FA_OK) return rc;
    fa::QuantParams p;
    p.x = static_cast<const __nv_bfloat16*>(x);
    p.out = static_cast<uint8_t*>(out);
    p.scales = scales;
    p.signs = signs;
    p.B = B;
    p.N = N;
    p.H = H;
    p.nb = static_cast<int>(nb);
    p.Np = static_cast<int>(fp8_vt_pitch(N));
    p.transpose = transpose ? 1 : 0;
    p.error_word = st->error_word;
    p.timeout_ns = g_fault_timeout_ns ? g_fault_timeout_ns : kDefaultTimeoutNs;
    CUtensorMap mx;
    if (make_map(&mx, x, rows, H, d, 128)) return FA_ERR_CUDA;
    // persistent: two CTAs per SM walk the blocks
    const int64_t nblocks = static_cast<int64_t>(B) * H * nb;
    const int grid = static_cast<int>(std::min<int64_t>(nblocks, 2 * static_cast<int64_t>(st->num_sms)));
    const int slot = prof_start(6, stream);
    if (transpose)
        fa::quantize_fp8_kernel<false, true><<<grid, fa::QuantCfg::THREADS, fa::QuantCfg::SMEM_BYTES, stream>>>(mx, p);
    else if (signs)
        fa::quantize_fp8_kernel<true, false><<<grid, fa::QuantCfg::THREADS, fa::QuantCfg::SMEM_BYTES, stream>>>(mx, p);
    else
        fa::quantize_fp8_kernel<false, false><<<grid, fa::QuantCfg::THREADS, fa::QuantCfg::SMEM_BYTES, stream>>>(mx, p);
    prof_stop(6, slot, stream);
    return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

int fa_fwd_fp8(const void* q8, const void* k8, const void* vt8, const float* sq, const float* sk,
               const float* sv, void* o, float* lse, int B, int H, int N, int d, float scale,
               int causal, int window, cudaStream_t stream) {
    if (!q8 || !k8 || !vt8 || !sq || !sk || !sv || !o || !lse) return FA_ERR_NULLPTR;
    if (d != 128) return FA_ERR_UNSUPPORTED_D;
    Common c;
    int rc = validate_common(B, H, N, d, scale, causal, window, nullptr, &c);
    if (rc != FA_OK) return rc;
    if (misaligned(q8) || misaligned(k8) || misaligned(vt8) || misaligned(o) || misaligned(lse) ||
        (reinterpret_cast<uintptr_t>(sq) & 3u) || (reinterpret_cast<uintptr_t>(sk) & 3u) ||
        (reinterpret_cast<uintptr_t>(sv) & 3u))
        return FA_ERR_MISALIGNED;
    if (B == 0 || c.rows == 0) return FA_OK;
    DeviceState* st = nullptr;
    if ((rc = device_setup(&st)) != FA_OK) return rc;
    CUtensorMap mq, mk, mv;
    if (make_map_u8_3d(&mq, q8, c.rows, H) || make_map_u8_3d(&mk, k8, c.rows, H) ||
        make_map_u8_2d(&mv, vt8, static_cast<int64_t>(B) * H * d, fp8_vt_pitch(N)))
        return FA_ERR_CUDA;
    fa::FwdParams p;
    p.g = c.g;
    p.o = static_cast<__nv_bfloat16*>(o);
    p.lse = lse;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.error_word = st->error_word;
    p.timeout_ns = g_fault_timeout_ns ? g_fault_timeout_ns : kDefaultTimeoutNs;
    p.fault_skip_v = 0;
    p.f8.sq = sq;
    p.f8.sk = sk;
    p.f8.sv = sv;
    p.nb = (N + 127) / 128;
    int grid = st->num_sms;
    const int64_t items = static_cast<int64_t>(B) * H * ((N + 255) / 256);
    if (items < grid) grid = static_cast<int>(items);
    using C8 = fa::FwdCfg<128, true>;
    const int slot = prof_start(7, stream);
    fa::fwd_kernel<128, true><<<grid, C8::THREADS, C8::SMEM_BYTES, stream>>>(mq, mk, mv, p);
    prof_stop(7, slot, stream);
    return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

size_t fa_bwd_workspace_size(int B, int H, int N, int d, int varlen_total) {
    (void)d;
    if (H <= 0 || B <= 0) return 0;
    const bool packed = varlen_total > 0;
    if (!packed && N <= 0) return 0;
    return fa::bwd_workspace_bytes(B, H, fa::bwd_stats_stride(B, N, varlen_total, packed), packed);
}

int fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
           const void* dO, void* dq, void* dk, void* dv, int B, int H, int N, int d, float scale,
           int causal, int window, const int* cu_seqlens, void* workspace, size_t workspace_bytes,
           cudaStream_t stream) {
    if (!q || !k || !v || !o || !lse || !dO || !dq || !dk || !dv) return FA_ERR_NULLPTR;
    Common c;
    int rc = validate_common(B, H, N, d, scale, causal, window, cu_seqlens, &c);
    if (rc != FA_OK) return rc;
    if (misaligned(q) || misaligned(k) || misaligned(v) || misaligned(o) || misaligned(lse) ||
        misaligned(dO) || misaligned(dq) || misaligned(dk) || misaligned(dv))
        return FA_ERR_MISALIGNED;
    if (B == 0 || c.rows == 0) return FA_OK;
    const bool packed = cu_seqlens != nullptr;
    const int64_t stride = fa::bwd_stats_stride(B, N, c.rows, packed);
    const size_t need = fa::bwd_workspace_bytes(B, H, stride, packed);
    if (!workspace || workspace_bytes < need) return FA_ERR_WORKSPACE;
    if (misaligned(workspace)) return FA_ERR_MISALIGNED;
    DeviceState* st = nullptr;
    if ((rc = device_setup(&st)) != FA_OK) return rc;

    fa::BwdArgs a;
    a.g = c.g;
    a.d = d;
    a.q = q;
    a.o = o;
    a.dO = dO;
    a.lse = lse;
    a.dq = dq;
    a.dk = dk;
    a.dv = dv;
    a.stats = static_cast<float*>(workspace);
    a.stats_stride = stride;
    a.scale = scale;
    a.num_sms = st->num_sms;
    a.error_word = st->error_word;
    a.timeout_ns = g_fault_timeout_ns ? g_fault_timeout_ns : kDefaultTimeoutNs;
    fa::BwdMaps m;
    if (make_map(&m.q, q, c.rows, H, d, 128) || make_map(&m.k, k, c.rows, H, d, 128) ||
        make_map(&m.v, v, c.rows, H, d, 128) || make_map(&m.dO, dO, c.rows, H, d, 128))
        return FA_ERR_CUDA;
    fa::BwdHooks hooks{prof_start, prof_stop};
    return fa::bwd_launch(a, m, stream, hooks) == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

size_t fa_bwd_fused_workspace_size(int B, int H, int N, int d, int varlen_total) {
    if (H <= 0 || B <= 0 || d != 128) return 0;
    const bool packed = varlen_total > 0;
    if (!packed && N <= 0) return 0;
    const int64_t rows = packed ? static_cast<int64_t>(varlen_total) : static_cast<int64_t>(B) * N;
    return fa::fused_workspace_bytes(B, H, fa::bwd_stats_stride(B, N, varlen_total, packed), packed,
                                     rows);
}

int fa_bwd_fused(const void* q, const void* k, const void* v, const void* o, const float* lse,
                 const void* dO, void* dq, void* dk, void* dv, int B, int H, int N, int d,
                 float scale, int causal, int window, const int* cu_seqlens, void* workspace,
                 size_t workspace_bytes, cudaStream_t stream) {
    if (!q || !k || !v || !o || !lse || !dO || !dq || !dk || !dv) return FA_ERR_NULLPTR;
    Common c;
    int rc = validate_common(B, H, N, d, scale, causal, window, cu_seqlens, &c);
    if (rc != FA_OK) return rc;
    if (d != 128) return FA_ERR_UNSUPPORTED_D;
    if (misaligned(q) || misaligned(k) || misaligned(v) || misaligned(o) || misaligned(lse) ||
        misaligned(dO) || misaligned(dq) || misaligned(dk) || misaligned(dv))
        return FA_ERR_MISALIGNED;
    if (B == 0 || c.rows == 0) return FA_OK;
    const bool packed = cu_seqlens != nullptr;
    const int64_t stride = fa::bwd_stats_stride(B, N, c.rows, packed);
    const size_t need = fa::fused_workspace_bytes(B, H, stride, packed, c.rows);
    if (!workspace || workspace_bytes < need) return FA_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return FA_ERR_MISALIGNED;
    DeviceState* st = nullptr;
    if ((rc = device_setup(&st)) != FA_OK) return rc;

    fa::BwdArgs a;
    a.g = c.g;
    a.d = d;
    a.q = q;
    a.o = o;
    a.dO = dO;
    a.lse = lse;
    a.dq = dq;
    a.dk = dk;
    a.dv = dv;
    a.stats = static_cast<float*>(workspace);
    a.stats_stride = stride;
    a.scale = scale;
    a.num_sms = st->num_sms;
    a.error_word = st->error_word;
    a.timeout_ns = g_fault_timeout_ns ? g_fault_timeout_ns : kDefaultTimeoutNs;
    float* dq_acc = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) +
                                             fa::fused_stats_bytes(B, H, stride, packed));
    fa::BwdMaps m;
    if (make_map(&m.q, q, c.rows, H, d, 128) || make_map(&m.k, k, c.rows, H, d, 128) ||
        make_map(&m.v, v, c.rows, H, d, 128) || make_map(&m.dO, dO, c.rows, H, d, 128))
        return FA_ERR_CUDA;
    fa::BwdHooks hooks{
        [](int kind, cudaStream_t s) { return prof_start(kind == 1 ? 1 : kind == 2 ? 8 : 9, s); },
        [](int kind, int slot, cudaStream_t s) { prof_stop(kind == 1 ? 1 : kind == 2 ? 8 : 9, slot, s); }};
    return fa::bwd_fused_launch(a, m, dq_acc, stream, hooks) == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

int fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const float* lse,
                   const void* dO, void* dq, void* dk, void* dv, int B, int H, int N, int d,
                   float scale, int causal, int window, const int* cu_seqlens,
                   cudaStream_t stream) {
    if (!q || !k || !v || !o || !lse || !dO || !dq || !dk || !dv) return FA_ERR_NULLPTR;
    Common c;
    int rc = validate_common(B, H, N, d, scale, causal, window, cu_seqlens, &c);
    if (rc != FA_OK) return rc;
    if (misaligned(q) || misaligned(k) || misaligned(v) || misaligned(o) || misaligned(lse) ||
        misaligned(dO) || misaligned(dq) || misaligned(dk) || misaligned(dv))
        return FA_ERR_MISALIGNED;
    if (B == 0 || c.rows == 0) return FA_OK;
    const bool packed = cu_seqlens != nullptr;
    const int64_t stride = fa::bwd_stats_stride(B, N, c.rows, packed);
    if (fa::bwd_workspace_bytes(B, H, stride, packed) > sizeof(float2) * FA_NOALLOC_MAX_ROWS)
        return FA_ERR_SCRATCH_LIMIT;
    DeviceState* st = nullptr;
    if ((rc = device_setup(&st)) != FA_OK) return rc;
    float2* scratch = nullptr;
    if ((rc = noalloc_setup(&scratch)) != FA_OK) return rc;

    fa::BwdArgs a;
    a.g = c.g;
    a.d = d;
    a.q = q;
    a.o = o;
    a.dO = dO;
    a.lse = lse;
    a.dq = dq;
    a.dk = dk;
    a.dv = dv;
    a.stats = reinterpret_cast<float*>(scratch);   // every entry the kernels use is written first by the pre-pass
    a.stats_stride = stride;
    a.scale = scale;
    a.num_sms = st->num_sms;
    a.error_word = st->error_word;
    a.timeout_ns = g_fault_timeout_ns ? g_fault_timeout_ns : kDefaultTimeoutNs;
    fa::BwdMaps m;
    if (make_map(&m.q, q, c.rows, H, d, 128) || make_map(&m.k, k, c.rows, H, d, 128) ||
        make_map(&m.v, v, c.rows, H, d, 128) || make_map(&m.dO, dO, c.rows, H, d, 128))
        return FA_ERR_CUDA;
    fa::BwdHooks hooks{prof_start, prof_stop};
    return fa::bwd_launch(a, m, stream, hooks) == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

const char* fa_status_string(int status) {
    switch (status) {
        case FA_OK: return "ok";
        case FA_ERR_NULLPTR: return "a required pointer is NULL";
        case FA_ERR_UNSUPPORTED_D: return "head dimension must be 64 or 128";
        case FA_ERR_BAD_SHAPE: return "invalid shape";
        case FA_ERR_MISALIGNED: return "a tensor pointer is not 16-byte aligned";
        case FA_ERR_BAD_MASK: return "a sliding window requires the causal mask";
        case FA_ERR_WORKSPACE: return "workspace missing or too small";
        case FA_ERR_CUDA: return "CUDA runtime or launch error";
        case FA_ERR_DEVICE_TIMEOUT: return "a bounded device-side wait timed out";
        case FA_ERR_BAD_SCALE: return "scale must be finite and positive";
        case FA_ERR_SCRATCH_LIMIT:
            return "problem exceeds the built-in scratch of fa_bwd_noalloc (use fa_bwd)";
        default: return "unknown status";
    }
}

int fa_get_device_error(cudaStream_t stream) {
    if (cudaStreamSynchronize(stream) != cudaSuccess) return FA_ERR_CUDA;
    DeviceState* st = nullptr;
    int rc = device_setup(&st);
    if (rc != FA_OK) return rc;
    int word = 0;
    if (cudaMemcpy(&word, st->error_word, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
        return FA_ERR_CUDA;
    if (word != 0) {
        const int zero = 0;
        if (cudaMemcpy(st->error_word, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess)
            return FA_ERR_CUDA;
        return FA_ERR_DEVICE_TIMEOUT;
    }
    return FA_OK;
}

int fa_profile_begin(void) {
    Profiler& P = g_prof;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_CUDA;
    if (P.created && P.device != dev) {
        for (int k = 0; k < kProfKinds; ++k)
            for (int i = 0; i < kProfCap; ++i) {
                cudaEventDestroy(P.ev[k][i][0]);
                cudaEventDestroy(P.ev[k][i][1]);
            }
        cudaFree(P.cta_clock);
        P.cta_clock = nullptr;
        P.created = false;
    }
    if (!P.created) {
        for (int k = 0; k < kProfKinds; ++k)
            for (int i = 0; i < kProfCap; ++i)
                if (cudaEventCreate(&P.ev[k][i][0]) != cudaSuccess ||
                    cudaEventCreate(&P.ev[k][i][1]) != cudaSuccess)
                    return FA_ERR_CUDA;
        // profiling only: the per-CTA timing buffer of the forward kernel
        if (cudaMalloc(&P.cta_clock, sizeof(unsigned long long) * (1 + 2 * kClockCtas)) != cudaSuccess ||
            cudaMemset(P.cta_clock, 0, sizeof(unsigned long long) * (1 + 2 * kClockCtas)) != cudaSuccess)
            return FA_ERR_CUDA;
        P.created = true;
        P.device = dev;
    }
    for (int k = 0; k < kProfKinds; ++k) P.n[k] = 0;
    if (cudaMemcpyToSymbol(fa::g_cta_clock, &P.cta_clock, sizeof(P.cta_clock)) != cudaSuccess)
        return FA_ERR_CUDA;
    P.on = true;
    return FA_OK;
}

int fa_profile_end(double* ms, int* counts) {
    Profiler& P = g_prof;
    P.on = false;
    unsigned long long* none = nullptr;
    if (P.created && cudaMemcpyToSymbol(fa::g_cta_clock, &none, sizeof(none)) != cudaSuccess)
        return FA_ERR_CUDA;
    for (int k = 0; k < kProfKinds; ++k) {
        double total = 0.0;
        for (int i = 0; i < P.n[k]; ++i) {
            if (cudaEventSynchronize(P.ev[k][i][1]) != cudaSuccess) return FA_ERR_CUDA;
            float t = 0.f;
            if (cudaEventElapsedTime(&t, P.ev[k][i][0], P.ev[k][i][1]) != cudaSuccess)
                return FA_ERR_CUDA;
            total += t;
        }
        if (ms) ms[k] = total;
        if (counts) counts[k] = P.n[k];
    }
    return FA_OK;
}

int fa_profile_cta_balance(double* balance, int* ctas) {
    Profiler& P = g_prof;
    if (!P.created || !P.cta_clock) return FA_ERR_CUDA;
    static unsigned long long h[1 + 2 * kClockCtas];
    if (cudaDeviceSynchronize() != cudaSuccess ||
        cudaMemcpy(h, P.cta_clock, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess)
        return FA_ERR_CUDA;
    const int G = static_cast<int>(h[0] < static_cast<unsigned long long>(kClockCtas) ? h[0] : kClockCtas);
    double sum = 0.0, mx = 0.0;
    for (int c = 0; c < G; ++c) {
        const double busy = static_cast<double>(h[2 + 2 * c] - h[1 + 2 * c]);
        sum += busy;
        if (busy > mx) mx = busy;
    }
    if (balance) *balance = (G > 0 && mx > 0.0) ? sum / G / mx : 0.0;
    if (ctas) *ctas = G;
    return FA_OK;
}

int fa_debug_set_fault(int mode, unsigned long long timeout_ns) {
    int prev = g_fault_mode;
    g_fault_mode = mode;
    g_fault_timeout_ns = timeout_ns;
    return prev;
}

}  // extern "C"
