// Internal declarations and device helpers of libhils (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "hils.h"

namespace hils {

constexpr int kChunk = 64;          // chunk size S (tokens per chunk)
constexpr unsigned kFull = 0xffffffffu;

typedef __nv_bfloat16 bf16;

// Time limits of the kernels' bounded waits (mbarrier phases of copies, tensor-core
// operations and other warps' hand-offs): a wait that runs past its limit sets the
// call's status word and the kernel stops, drains what it started and returns.
constexpr long long kWaitLimitNs = 100ll * 1000 * 1000;   // waits on work in progress
constexpr long long kDrainLimitNs = 100ll * 1000 * 1000;  // waits for a stopped CTA's own copies and MMAs
// The work-wait limit of a call: zero under HILS_FLAG_DIAG_EXPIRE_WAITS (diagnostic).
inline long long work_wait_ns(uint32_t flags) { return (flags & HILS_FLAG_DIAG_EXPIRE_WAITS) ? 0 : kWaitLimitNs; }

// ------------------------------------------------------------------ launch args

// Strided [B, H, T, d] view in elements.
struct View {
    const void *ptr;
    int64_t sb, sh, st;
};
struct MutView {
    void *ptr;
    int64_t sb, sh, st;
};

struct SummarizeArgs {
    View K, LQ;
    MutView Ksum;
    float *Bsum;
    int B, H, C;
    float scale;
    int G = 1;             // query heads per key-value head: K has H / G heads
    const int32_t *cache_len = nullptr;  // non-null: only the chunk each sequence's newest token completed
};

struct SelectArgs {
    View Qcal, Ksum;
    const float *Bsum;
    const int32_t *qpos;   // [B, Lq] or null (t = i)
    int qpos_bias;         // added to qpos (-1 when qpos holds decode cache lengths)
    int32_t *idx;
    float *score;
    int32_t *nsel;
    int B, H, Lq, C, topk;
    float scale;
    int path;              // SelectPath chosen by select_plan
    int G = 1;             // query heads per group: idx and nsel have H / G heads
    int excl_w = 0;        // > 0: the window length; chunks wholly inside a query's window are not eligible
    // split search over chunk ranges (decode-like shapes)
    int ctas_per_query;    // summary blocks per query of the screen kernel
    int tiles_per_warp;    // 128-chunk tiles each warp scans
    void *ws;              // status word, then the screen values of the split search
    long long wait_ns = kWaitLimitNs;  // limit of a bounded wait on work in progress (0: expire at once)
};

// Which select kernels run: one warp per query; screen + pick (few queries, long
// tables); tensor-core scoring with one thread per query (many bf16 queries, d = 128).
// Groups of G > 1 heads: one warp per (b, group, query) over all of the group's heads.
constexpr int kMaxGroupHeads = 8;  // query heads per key-value head supported (H / H_kv)
enum SelectPath { kSelectWarp = 0, kSelectSplit = 1, kSelectTc = 2, kSelectGroup = 3 };
constexpr size_t kSelectStatusBytes = 256;  // status word at the front of the select workspace

struct AttendArgs {
    View Q, K, V;
    MutView O;
    float *lse;            // [B, H, Lq] or null
    const int32_t *idx;    // [B, H / G, Lq, Ksel]
    const float *score;    // [B, H, Lq, Ksel]
    const int32_t *nsel;   // [B, H / G, Lq]
    const int32_t *qpos;   // prefill: null (t = i); decode: null and cache_len set
    const int32_t *cache_len;  // decode: [B]
    int B, H, Lq, topk, W;
    float scale;
    int units;             // units per query: K chunk units + window tiles
    int window_early;      // decode: window tiles may start before the preceding grid ends
    void *ws;
    int G = 1;             // query heads per key-value head: K, V, idx and nsel have H / G heads
    long long wait_ns = kWaitLimitNs;  // limit of a bounded wait on work in progress (0: expire at once)
};

// Host launchers (one translation unit each). They return HILS_OK or HILS_ERR_CUDA.
// Backward pass (fixed selection; float32 dense gradients, the shared ones accumulated).

hils_status launch_summarize(hils_dtype dt, int d, const SummarizeArgs &a, cudaStream_t s);
hils_status launch_select(hils_dtype dt, int d, const SelectArgs &a, cudaStream_t s);
hils_status launch_attend_decode(hils_dtype dt, int d, const AttendArgs &a, cudaStream_t s);
hils_status launch_attend_prefill_general(hils_dtype dt, int d, const AttendArgs &a, cudaStream_t s);
// Tensor-core prefill (bf16, d = 128): used when supported; `status` receives a nonzero
// word if one of its bounded waits expired.
bool attend_prefill_tc_supported(hils_dtype dt, int d, int N);
hils_status launch_attend_prefill_tc(const AttendArgs &a, int N, uint32_t *status, cudaStream_t s);
constexpr size_t kPrefillWsBytes = 256;  // status word (+ padding)

// Workspace layouts (bytes); shared by the host size query and the kernels.
size_t select_ws_bytes(int queries, int C, int path);
size_t attend_decode_ws_bytes(int queries, int units, int d);
// Leading part of the decode attend workspace that must start at zero (one arrival
// counter per query, rounded to 256 bytes); every call leaves it zero.
__host__ __device__ inline size_t attend_decode_counter_bytes(int queries) {
    return ((size_t)queries * sizeof(int) + 255) & ~(size_t)255;
}

// Choice of the select kernels (path, ctas_per_query, tiles_per_warp of `a`); the
// workspace size depends only on the sizes, never on has_qpos, so the size query and
// the call agree.
void select_plan(hils_dtype dt, int d, int B, int H, int Lq, int C, int K, bool has_qpos, int num_sms,
                 SelectArgs *a);
// Tensor-core select (bf16, d = 128, at most 512 eligible chunks per query).
bool select_tc_supported(hils_dtype dt, int d, int B, int H, int Lq, int C, int K, bool has_qpos, int G);
hils_status launch_select_tc(const SelectArgs &a, cudaStream_t s);

int device_sm_count();
// The argument checks of hils_attend_decode (parameters, views, arrays), without launching.
int check_attend_decode_args(const hils_params *p, hils_ctensor Q, hils_ctensor Kc, hils_ctensor Vc,
                             const int32_t *cache_len, const int32_t *idx, const float *score, const int32_t *nsel,
                             hils_tensor O, float *lse);
hils_status record_cuda_error(cudaError_t e);

// Per-kernel launch set-up done once per device: the dynamic shared memory opt-in and
// the resident CTAs per SM. `cache` is a function-local static of the caller.
struct KernelSetup {
    unsigned long long done = 0;  // bit per device ordinal < 64
    int per_sm[64] = {};
};
hils_status kernel_setup(KernelSetup &cache, const void *func, int threads, int smem_bytes, int *per_sm);

// Launches `func(args)` with programmatic stream serialization: the kernel may be
// scheduled while the previous kernel on the stream drains, and must call pdl_wait()
// before touching anything that kernel (or earlier work) writes.
template <typename Args>
hils_status launch_dependent(const void *func, dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                             const Args &args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    void *argv[] = {const_cast<Args *>(&args)};
    return record_cuda_error(cudaLaunchKernelExC(&cfg, func, argv));
}

// ------------------------------------------------------------------ device helpers

// Programmatic dependent launch: wait for the preceding grid's completion (and its
// memory), and allow the next dependent-launched grid to be scheduled.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Nanoseconds of the GPU's global timer: the clock of every bounded wait.
__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" :::); }

template <typename T>
struct Vec;  // one 16-byte vector of T
template <>
struct Vec<float> {
    static constexpr int kN = 4;
};
template <>
struct Vec<bf16> {
    static constexpr int kN = 8;
};

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Widens the 16 bytes `v` into Vec<T>::kN floats.
__device__ __forceinline__ void widen(const uint4 &v, float (&f)[8], bf16) {
    f[0] = bf16lo(v.x); f[1] = bf16hi(v.x);
    f[2] = bf16lo(v.y); f[3] = bf16hi(v.y);
    f[4] = bf16lo(v.z); f[5] = bf16hi(v.z);
    f[6] = bf16lo(v.w); f[7] = bf16hi(v.w);
}
__device__ __forceinline__ void widen(const uint4 &v, float (&f)[4], float) {
    f[0] = __uint_as_float(v.x); f[1] = __uint_as_float(v.y);
    f[2] = __uint_as_float(v.z); f[3] = __uint_as_float(v.w);
}

// Sum of the element-wise products of two 16-byte vectors of T, added to acc.
template <typename T>
__device__ __forceinline__ float dot16(const uint4 &a, const uint4 &b, float acc) {
    float fa[Vec<T>::kN], fb[Vec<T>::kN];
    widen(a, fa, T());
    widen(b, fb, T());
#pragma unroll
    for (int i = 0; i < Vec<T>::kN; ++i) acc = fmaf(fa[i], fb[i], acc);
    return acc;
}

// Two adjacent elements of T widened to float.
__device__ __forceinline__ float2 load2(const bf16 *p) {
    const uint32_t w = *reinterpret_cast<const uint32_t *>(p);
    return make_float2(bf16lo(w), bf16hi(w));
}
__device__ __forceinline__ float2 load2(const float *p) { return *reinterpret_cast<const float2 *>(p); }

// Two floats rounded to T (nearest-even) and stored.
__device__ __forceinline__ void store2(bf16 *p, float a, float b) {
    *reinterpret_cast<__nv_bfloat162 *>(p) = __floats2bfloat162_rn(a, b);
}
__device__ __forceinline__ void store2(float *p, float a, float b) {
    *reinterpret_cast<float2 *>(p) = make_float2(a, b);
}

__device__ __forceinline__ double to_double(bf16 x) { return (double)__bfloat162float(x); }
__device__ __forceinline__ double to_double(float x) { return (double)x; }

__device__ __forceinline__ void cp_async16(void *smem, const void *gmem) {
    const unsigned s = (unsigned)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, o));
    return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
    return v;
}

// Monotone map of a float onto unsigned ints (larger float -> larger key); finite
// floats and -inf map to keys > 0, so 0 can mean "no element".
__device__ __forceinline__ unsigned ordered_key(float f) {
    const unsigned b = __float_as_uint(f);
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float key_to_float(unsigned k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

}  // namespace hils
