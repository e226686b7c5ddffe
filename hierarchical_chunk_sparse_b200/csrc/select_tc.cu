// Chunk scores and exact top-K for many queries on the 5th-generation tensor cores:
// "Hierarchical Sparse Attention Done Right" (picx.dev summary), Eq. 7 and
// Methodology 2, and the rcap.io post's pseudocode figure (keep the top K chunks per
// query). bf16, d = 128, at most 512 eligible chunks per query.
//
// One CTA of 128 threads takes 128 consecutive queries of one (b, h); thread r owns
// query row r, which is also TMEM lane r.
//   1. TMA brings the query tile (128 x 128 bf16) and the head's first nc summary rows
//      (nc = the CTA's largest eligible count, rounded up to 64) into shared memory
//      with the 128-byte swizzle; one thread issues S = Q~ K'^T (M = 128, N <= 256 per
//      instruction, eight K-steps of 16) into TMEM as float32.
//   2. Each thread reads its row of S back from TMEM 32 columns at a time and forms
//      the screen values s_c = fma(S_c, scale, b'_c) with the radius
//        e_c = scale |q~| |k'_c| d 2^-16 (1 + 2^-8) + |s_c| 2^-22,
//      the bound that leaves room for any order and rounding of the tensor core's
//      float32 accumulation (about 2^7 times the round-to-nearest bound).
//      e_max (an upper bound on every e_c of the row) comes from the row's largest
//      |k'| and |s|.
//   3. Candidates: a threshold guess g from the row's mean and spread (normal fit for
//      about K + 4 values above it) sets the cut t = g - 2 e_max, and one pass collects
//      every chunk with s >= t, in ascending chunk order. The list certifies itself
//      when it holds at least K and at most 32 entries and t <= s_K - 2 e_max (s_K =
//      the list's K-th largest value): every chunk left out then has
//      s + e < s_K - e_max <= lo of each of the K largest, so it is certainly out.
//      Otherwise the guess moves (bisection, or g = s_K) and the pass repeats.
//   4. On the list: s_K and s_{K+1}; chunks with lo > s_{K+1} + e_max are certainly in,
//      chunks with hi < s_K - e_max certainly out, and when the in-set leaves places
//      open among several remaining ("band") chunks, those get the float64 score,
//      computed by the whole CTA from a shared work list. The kept list is written in
//      ascending chunk index with the float32 screen values.
// Rows whose candidates or band entries exceed the list capacity (heavy ties) are
// finished by the warp routine of the other select kernels, which is exact for any
// input. Every mbarrier wait is bounded; on expiry the CTA sets the status word,
// waits (bounded) for the copies and MMAs it started, frees its TMEM and writes no
// output.
//
// Grouped heads (summary page, Methodology 3, GQA adaptation): a CTA takes 128 queries
// of one (b, group) and puts S_h = Q~_h K'_h^T of each of the group's G heads into its
// own TMEM columns (the heads' operands pass through two shared-memory buffers). A
// chunk's group value is the maximum over the heads of s_h,c. Once the MMAs are done,
// one pass folds the heads' intervals s_h,c +- e_h,c into [max lo, max hi] per chunk
// and keeps the centre in shared memory (in the operand buffers, which the MMAs no
// longer read); every later pass reads the centres, and every chunk takes the row's
// largest folded radius e_max as its radius (an upper bound on its own), so the steps
// above apply unchanged. The band's float64 score is the largest of the heads' float64
// scores, and each head's output score of a kept chunk is its own screen value, read
// back from its columns.
#include "select_common.cuh"
#include "tc_common.cuh"

namespace hils {
namespace {

using namespace tc;

constexpr int kQM = 128;           // queries per CTA (TMEM lanes)
constexpr int kHD = 128;           // head dimension
constexpr int kTcThreads = 128;
constexpr int kMaxCols = 512;      // TMEM columns: eligible chunks per CTA times the heads
constexpr int kCap = 32;           // candidate slots per query (one spare slot absorbs overflow)
constexpr int kBandCap = 8;        // float64 rescoring slots per query
constexpr int kCollectPasses = 6;
constexpr int kQBytes = 2 * kQM * 128;  // one head's query tile: 2 column blocks x 128 rows x 128 B

// Reused region (after the MMAs have read the operands): per-thread candidate lists,
// band scores, the CTA's work list and the fallback's scratch.
constexpr int kListS = 0;                                  // float  [kCap + 1][128]
constexpr int kListC = kListS + (kCap + 1) * kQM * 4;      // uint16 [kCap + 1][128]
constexpr int kBandX = kListC + (kCap + 1) * kQM * 2;      // double [kBandCap][128]
constexpr int kBandJ = kBandX + kBandCap * kQM * 8;        // uint8  [kBandCap][128]
constexpr int kWork = kBandJ + kBandCap * kQM;             // uint16 [128 * kBandCap]
constexpr int kFbQ = kWork + kQM * kBandCap * 2;           // float  [4][128]
constexpr int kFbList = kFbQ + 4 * kHD * 4;                // EntryList [4]
constexpr int kReuseBytes = kFbList + 4 * kListBytes;
// grouped heads: the fallback needs the query rows of all the group's heads, and the
// folded centre of every (chunk, row) follows
constexpr int kFbQG = kReuseBytes;                         // float  [4][kMaxGroup][128]
constexpr int kFold = kFbQG + 4 * kMaxGroup * kHD * 4;     // float  [ncpad][128]
static_assert(kBandX % 8 == 0 && kFbList % 8 == 0 && kFold % 16 == 0, "alignment");
static_assert(kReuseBytes <= kQBytes + 2 * 64 * 128, "reused region fits the smallest operand area");
// two operand buffers of kQBytes + 2 * ncpad * 128 bytes each hold kFold + ncpad * 128 * 4
static_assert(kFold <= 2 * kQBytes, "grouped reused region and folded centres fit two operand buffers");

struct Misc {
    unsigned long long bar[5];  // operands loaded (2 buffers), MMAs read a buffer (2), all MMAs done
    uint32_t tmem;
    uint32_t abort;
    int nc;
    uint32_t knmax;             // float bits of the largest |k'_c|, c < nc
    int nwork;
    int novf;
    uint8_t ovf[kQM];
};

// Shared memory: nbuf operand buffers (a head's query tile, then its first ncpad summary
// rows, both as 2 column blocks with the 128-byte swizzle), then per head the biases,
// norms and magnitude ranges of its summary rows and of the query rows.
struct Layout {
    int buf, nbuf, bias, kn, kmag, qmag, qn, misc, total;
};
__host__ __device__ inline Layout layout(int ncpad, int G) {
    Layout L;
    L.buf = kQBytes + 2 * ncpad * 128;
    L.nbuf = G < 2 ? G : 2;
    L.bias = L.nbuf * L.buf;               // float [G][ncpad]
    L.kn = L.bias + G * ncpad * 4;         // float [G][ncpad]
    L.kmag = L.kn + G * ncpad * 4;         // uint32 [G][ncpad]: smallest nonzero | largest magnitude << 16
    L.qmag = L.kmag + G * ncpad * 4;       // uint32 [G][128], as kmag for the query rows
    L.qn = L.qmag + G * kQM * 4;           // float [G][128]
    L.misc = L.qn + G * kQM * 4;
    L.total = L.misc + (int)sizeof(Misc);
    return L;
}

struct TcSelArgs {
    SelectArgs a;
    int ncpad;      // summary rows staged per CTA and head at most (multiple of 64)
    uint32_t hcols; // TMEM columns per head (power of two >= ncpad)
    uint32_t cols;  // TMEM columns allocated (power of two >= G * hcols)
    uint32_t *status;
};

// |v|^2 of a 128-element bf16 row stored as two 128-byte-swizzled column blocks, and
// its magnitude range: smallest nonzero | largest bf16 magnitude << 16 (0xffff: none).
__device__ __forceinline__ float row_stats(const uint8_t *blk0, int block_stride, int r, uint32_t &mag) {
    float acc = 0.f;
    uint32_t mlo = 0xffffu, mhi = 0u;
#pragma unroll
    for (int kb = 0; kb < 2; ++kb) {
        const uint8_t *row = blk0 + kb * block_stride + r * 128;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const uint4 v = *reinterpret_cast<const uint4 *>(row + ((u ^ (r & 7)) << 4));
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int p = 0; p < 4; ++p) {
                const float lo = bf16lo(w[p]), hi = bf16hi(w[p]);
                acc = fmaf(lo, lo, fmaf(hi, hi, acc));
                const uint32_t a0 = w[p] & 0x7fffu, a1 = (w[p] >> 16) & 0x7fffu;
                mhi = max(mhi, max(a0, a1));
                mlo = min(mlo, min(a0 ? a0 : 0xffffu, a1 ? a1 : 0xffffu));
            }
        }
    }
    mag = mlo | mhi << 16;
    return acc;
}

__device__ __forceinline__ float bf16_mag(uint32_t m) { return __uint_as_float(m << 16); }

// True when every product q_x k_x of the two rows is exact in float32: each nonzero
// product lies in [2^-126, 2^127) (a product of two bf16 values has at most 16
// significant bits), or one row is zero. Then the float64 chain below, fed with the
// float32 products, equals the one fed with float64 products.
__device__ __forceinline__ bool products_exact_f32(uint32_t qm, uint32_t km) {
    const uint32_t qlo = qm & 0xffffu, qhi = qm >> 16, klo = km & 0xffffu, khi = km >> 16;
    if (qhi == 0u || khi == 0u) return true;
    const double pmin = (double)bf16_mag(qlo) * (double)bf16_mag(klo);
    const double pmax = (double)bf16_mag(qhi) * (double)bf16_mag(khi);
    return pmin >= 0x1p-126 && pmax < 0x1p127;  // NaN or inf magnitudes fail the second test
}

// The float64 score x_c = (sum_x q~_x k'_x) * scale + b'_c with every product formed
// exactly in float32 (see products_exact_f32), then summed in x order in float64.
__device__ double exact_score_f32prod(const bf16 *qrow, const bf16 *krow, float scale, float bias) {
    const uint4 *qr = reinterpret_cast<const uint4 *>(qrow);
    const uint4 *kr = reinterpret_cast<const uint4 *>(krow);
    double acc = 0.0;
#pragma unroll
    for (int hlf = 0; hlf < 2; ++hlf) {
        uint4 qv[8], kv[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            qv[u] = __ldg(qr + hlf * 8 + u);
            kv[u] = __ldg(kr + hlf * 8 + u);
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const uint32_t qw[4] = {qv[u].x, qv[u].y, qv[u].z, qv[u].w};
            const uint32_t kw[4] = {kv[u].x, kv[u].y, kv[u].z, kv[u].w};
#pragma unroll
            for (int p = 0; p < 4; ++p) {
                acc = __dadd_rn(acc, (double)__fmul_rn(bf16lo(qw[p]), bf16lo(kw[p])));
                acc = __dadd_rn(acc, (double)__fmul_rn(bf16hi(qw[p]), bf16hi(kw[p])));
            }
        }
    }
    return __dadd_rn(__dmul_rn(acc, (double)scale), (double)bias);
}

template <bool kGroup>
__global__ void __launch_bounds__(kTcThreads) select_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                                                                const __grid_constant__ CUtensorMap tmK,
                                                                TcSelArgs args) {
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte alignment by pointer arithmetic on the shared array, so that the compiler
    // keeps every access below in the shared address space
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const SelectArgs &a = args.a;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = kGroup ? a.G : 1;
    const int i0 = blockIdx.x * kQM;
    const int units = a.H / G;                                   // heads, or groups, per batch
    const int b = blockIdx.y / units, h0 = (blockIdx.y % units) * G;  // the CTA's first query head
    const int K = a.topk;
    const int ncpad = args.ncpad;
    const Layout L = layout(ncpad, G);
    const uint32_t sbase = smem_u32(smem);
    float *bias_s = reinterpret_cast<float *>(smem + L.bias);
    float *kn_s = reinterpret_cast<float *>(smem + L.kn);
    uint32_t *kmag_s = reinterpret_cast<uint32_t *>(smem + L.kmag);
    uint32_t *qmag_s = reinterpret_cast<uint32_t *>(smem + L.qmag);
    float *qn_s = reinterpret_cast<float *>(smem + L.qn);
    Misc *misc = reinterpret_cast<Misc *>(smem + L.misc);
    const uint32_t bar_load[2] = {smem_u32(&misc->bar[0]), smem_u32(&misc->bar[1])};
    const uint32_t bar_read[2] = {smem_u32(&misc->bar[2]), smem_u32(&misc->bar[3])};
    const uint32_t bar_done = smem_u32(&misc->bar[4]);

    // ---- positions; the CTA's eligible range
    const int i = i0 + tid;
    const bool row_ok = i < a.Lq;
    int t = -1;
    if (row_ok) t = a.qpos ? a.qpos[(int64_t)b * a.Lq + i] + a.qpos_bias : i;
    const int ne = row_ok ? eligible(t, a.C, a.excl_w) : 0;
    if (tid == 0) {
        misc->nc = 0;
        misc->knmax = 0u;
        misc->nwork = 0;
        misc->novf = 0;
        misc->abort = 0u;
        for (int k = 0; k < 5; ++k) mbar_init(smem_u32(&misc->bar[k]), 1);
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    __syncthreads();
    const int ne_w = __reduce_max_sync(kFull, ne);
    if (lane == 0) atomicMax(&misc->nc, ne_w);
    __syncthreads();
    const int nc = misc->nc;  // uniform
    const int nrows = (nc + 63) & ~63;

    volatile uint32_t *abort_flag = &misc->abort;
    // bounded wait on work in progress (a.wait_ns of the global timer; zero, a diagnostic:
    // every such wait expires at once)
    auto wait = [&](uint32_t barrier, uint32_t parity) {
        if (*abort_flag) return false;
        if (a.wait_ns > 0) {
            if (mbar_try_wait(barrier, parity)) return true;
            const uint64_t t0 = global_ns();
            for (int it = 0;; ++it) {
                if (mbar_try_wait(barrier, parity)) return true;
                if ((it & 15) == 15 && (long long)(global_ns() - t0) > a.wait_ns) break;
            }
        }
        *abort_flag = 1u;
        atomicOr(args.status, 1u);
        return false;
    };
    auto drain_wait = [&](uint32_t barrier, uint32_t parity) {  // this CTA's own copies and MMAs
        const uint64_t t0 = global_ns();
        while (!mbar_try_wait(barrier, parity))
            if ((long long)(global_ns() - t0) > kDrainLimitNs) break;
    };

    // thread 0's record of what it started: loads per buffer, MMAs, the final commit
    int loads[2] = {0, 0};
    bool issued_mma = false, committed = false;
    auto issue_load = [&](int hh) {  // head hh's operands into buffer hh & 1 (thread 0)
        const int bf = hh & 1;
        const uint32_t dst = sbase + bf * L.buf;
        ++loads[bf];
        mbar_expect_tx(bar_load[bf], kQBytes + 2 * nrows * 128);
        tma_load_4d(dst, &tmQ, bar_load[bf], 0, i0, h0 + hh, b);
        tma_load_4d(dst + 16384, &tmQ, bar_load[bf], 64, i0, h0 + hh, b);
        for (int r0 = 0; r0 < nrows; r0 += 64) {
            tma_load_4d(dst + kQBytes + r0 * 128, &tmK, bar_load[bf], 0, r0, h0 + hh, b);
            tma_load_4d(dst + kQBytes + ncpad * 128 + r0 * 128, &tmK, bar_load[bf], 64, r0, h0 + hh, b);
        }
    };
    if (nc > 0) {
        if (warp == 0) {
            asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(
                             smem_u32(&misc->tmem)),
                         "r"(args.cols));
            asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n");
        }
        if (tid == 0)
            for (int hh = 0; hh < L.nbuf; ++hh) issue_load(hh);
        for (int hh = 0; hh < G; ++hh) {
            const float *bhead = a.Bsum + ((int64_t)b * a.H + h0 + hh) * a.C;
            for (int c = tid; c < nc; c += kTcThreads) bias_s[hh * ncpad + c] = __ldg(bhead + c);
        }
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    }
    const uint32_t tmem = nc > 0 ? misc->tmem : 0u;

    // ---- per head: operands in shared memory, their norms, then S_h = Q~_h K'_h^T into
    // TMEM columns [hh * hcols, hh * hcols + nrows)
    if (nc > 0) {
        for (int hh = 0; hh < G; ++hh) {
            const int bf = hh & 1;
            const uint32_t ph = (uint32_t)(hh >> 1) & 1u;
            const uint8_t *buf = smem + bf * L.buf;
            if (wait(bar_load[bf], ph)) {
                float knm = 0.f;
                for (int c = tid; c < nc; c += kTcThreads) {
                    uint32_t km;
                    const float kn = sqrtf(row_stats(buf + kQBytes, ncpad * 128, c, km));
                    kn_s[hh * ncpad + c] = kn;
                    kmag_s[hh * ncpad + c] = km;
                    knm = fmaxf(knm, kn);
                }
                if (!kGroup) {
                    knm = warp_max(knm);
                    if (lane == 0) atomicMax(&misc->knmax, __float_as_uint(knm));  // non-negative floats order as integers
                }
                uint32_t qm;
                qn_s[hh * kQM + tid] = sqrtf(row_stats(buf, 16384, tid, qm));
                qmag_s[hh * kQM + tid] = qm;
                if (tid == 0 && !*abort_flag) {
                    tc_fence_after();
                    const uint32_t ob = sbase + bf * L.buf;
                    const int nblk = (nrows + 255) / 256;
                    for (int nb = 0; nb < nblk; ++nb) {
                        const int n = min(256, nrows - nb * 256);
                        const uint32_t idesc = idesc_bf16(kQM, n, false);
#pragma unroll
                        for (int ks = 0; ks < kHD / 16; ++ks) {
                            const uint32_t qa = ob + (ks >> 2) * 16384 + (ks & 3) * 32;
                            const uint32_t ka = ob + kQBytes + (ks >> 2) * (ncpad * 128) + nb * 256 * 128 + (ks & 3) * 32;
                            mma_ss(tmem + hh * args.hcols + nb * 256, smem_desc(qa, 16, 1024), smem_desc(ka, 16, 1024),
                                   idesc, ks > 0);
                        }
                    }
                    issued_mma = true;
                    if (hh + 2 < G) mma_commit(bar_read[bf]);
                    if (hh == G - 1) {
                        mma_commit(bar_done);
                        committed = true;
                    }
                }
            }
            if (hh + 2 < G) {  // reload buffer bf with head hh + 2 once its MMAs have read it
                __syncthreads();  // every thread's norms of head hh are done
                if (tid == 0 && issued_mma && !*abort_flag && wait(bar_read[bf], ph)) issue_load(hh + 2);
            }
        }
    }
    __syncthreads();
    if (nc > 0) wait(bar_done, 0);
    tc_fence_after();
    __syncthreads();
    if (*abort_flag) {  // uniform: read after the barrier
        if (tid == 0) {  // let every started copy and MMA complete before leaving
            for (int bf = 0; bf < 2; ++bf) {
                if (loads[bf] == 0) continue;  // each load was issued after the previous one of its buffer completed
                drain_wait(bar_load[bf], (uint32_t)(loads[bf] - 1) & 1u);
            }
            if (issued_mma) {
                if (!committed) mma_commit(bar_done);
                drain_wait(bar_done, 0);
            }
        }
        tc_fence_before();
        __syncthreads();
        if (nc > 0 && warp == 0) {
            tc_fence_after();
            asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(args.cols));
        }
        return;
    }

    // ---- per-row selection (thread = query row = TMEM lane)
    float *ls = reinterpret_cast<float *>(smem + kListS);
    uint16_t *lc = reinterpret_cast<uint16_t *>(smem + kListC);
    double *bx = reinterpret_cast<double *>(smem + kBandX);
    uint8_t *bj_s = smem + kBandJ;
    uint16_t *work = reinterpret_cast<uint16_t *>(smem + kWork);
    const float sc = a.scale;
    const float eq = sc * qn_s[tid] * ((float)kHD * 0x1p-16f) * (1.f + 0x1p-8f);
    const float knmax = __uint_as_float(misc->knmax);
    const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
    const int nbat = (ne_w + 31) >> 5;  // warp-uniform: tcgen05.ld is warp-collective
    // grouped heads: fold the heads' intervals of every eligible chunk once; the centre
    // goes to shared memory, the largest radius of the row to emx
    float *fold = reinterpret_cast<float *>(smem + kFold);  // [chunk][row]
    float emx = 0.f;
    if constexpr (kGroup) {
        for (int bi = 0; bi < nbat; ++bi) {
            float lo[32], hi[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) lo[j] = hi[j] = -INFINITY;
            for (int hh = 0; hh < G; ++hh) {
                uint32_t r[32];
                tmem_ld32(trow + hh * args.hcols + bi * 32, r);
                tmem_wait_ld();
                const float eqh = sc * qn_s[hh * kQM + tid] * ((float)kHD * 0x1p-16f) * (1.f + 0x1p-8f);
                const float *bh = bias_s + hh * ncpad + bi * 32;
                const float *kh = kn_s + hh * ncpad + bi * 32;
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    if (bi * 32 + j < ne) {
                        const float sh = fmaf(__uint_as_float(r[j]), sc, bh[j]);
                        fold_interval(sh, fmaf(eqh, kh[j], fabsf(sh) * 0x1p-22f), lo[j], hi[j]);
                    }
                }
            }
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const int c = bi * 32 + j;
                if (c < ne) {
                    float s, e;
                    interval_mid(lo[j], hi[j], s, e);
                    fold[c * kQM + tid] = s;
                    emx = fmaxf(emx, e);
                }
            }
        }
    }
    // f(c, s) over this row's eligible chunks, ascending
    auto for_each = [&](auto &&f) {
        if constexpr (!kGroup) {
            for (int bi = 0; bi < nbat; ++bi) {
                uint32_t r[32];
                tmem_ld32(trow + bi * 32, r);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int c = bi * 32 + j;
                    if (c < ne) f(c, fmaf(__uint_as_float(r[j]), sc, bias_s[c]));
                }
            }
        } else {
#pragma unroll 8
            for (int c = 0; c < ne; ++c) f(c, fold[c * kQM + tid]);
        }
    };

    // pass A: range and moments of the row (shifted by b'_0, which lies near every s)
    const float sref = nc > 0 ? bias_s[0] : 0.f;
    float mn = INFINITY, mx = -INFINITY, sum = 0.f, sq = 0.f;
    for_each([&](int, float s) {
        mn = fminf(mn, s);
        mx = fmaxf(mx, s);
        const float dv = s - sref;
        sum += dv;
        sq = fmaf(dv, dv, sq);
    });
    const float emax = kGroup ? emx : fmaf(eq, knmax, fmaxf(fabsf(mn), fabsf(mx)) * 0x1p-22f);

    // candidate list: collect s >= tcut; certify or move the guess g and collect again
    float g = -INFINITY;  // -inf: take every eligible chunk (rows with ne <= K + 4)
    float lo_g = mn, hi_g = INFINITY;  // counts above lo_g too large, above hi_g too small
    if (ne > K + 4) {
        const float mu = sum / (float)ne;
        const float sd = sqrtf(fmaxf(sq / (float)ne - mu * mu, 0.f));
        const float p = ((float)K + 4.f) / (float)ne;  // upper-tail share to keep, < 1
        const float z = p <= 0.5f ? normal_upper_quantile(p) : -normal_upper_quantile(1.f - p);
        g = fminf(fmaxf(sref + mu + sd * z, mn), mx);
    }
    bool pending = true;
    int m = 0;
    float sK = 0.f, sK1 = 0.f;
    uint32_t alive = 0u;  // after certification: the entries not among the m - K smallest
    for (int pass = 0; pass < kCollectPasses && __any_sync(kFull, pending); ++pass) {
        const float tcut = g == -INFINITY ? -INFINITY : __fsub_rd(__fsub_rd(g, emax), emax);
        int mm = 0;
        for_each([&](int c, float s) {
            const bool take = pending && s >= tcut;
            const int slot = min(mm, kCap);  // entries past the capacity land in the spare slot
            if (take) {
                ls[slot * kQM + tid] = s;
                lc[slot * kQM + tid] = (uint16_t)c;
            }
            mm += take ? 1 : 0;
        });
        if (!pending) continue;
        m = mm;
        if (m > kCap) {  // cut too low: raise the guess
            lo_g = g;
            g = 0.5f * (g + fminf(hi_g, mx));
            continue;
        }
        // the m - K smallest leave (the last one is s_{K+1}); the smallest left is s_K
        alive = m == 32 ? ~0u : ((1u << m) - 1u);
        for (int r = 0; r < m - K; ++r) {
            float best = INFINITY;
            int bj = 0;
            uint32_t bit = 1u;
            for (int j = 0; j < m; ++j, bit <<= 1) {
                const float v = ls[j * kQM + tid];
                if ((alive & bit) && v < best) {
                    best = v;
                    bj = j;
                }
            }
            alive &= ~(1u << bj);
            sK1 = best;
        }
        sK = INFINITY;
        for (int j = 0; j < m; ++j)
            if (alive >> j & 1u) sK = fminf(sK, ls[j * kQM + tid]);
        if (g == -INFINITY || (m >= K && tcut <= __fsub_rd(__fsub_rd(sK, emax), emax))) {
            pending = false;  // certified
        } else if (m >= K) {
            g = sK;  // the exact K-th largest: the next cut certifies unless it admits too many
        } else {  // fewer than K above the cut: lower the guess
            hi_g = g;
            g = 0.5f * (lo_g + g);
        }
    }
    auto free_tmem = [&]() {
        tc_fence_before();
        __syncthreads();
        if (nc > 0 && warp == 0) {
            tc_fence_after();
            asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(args.cols));
        }
    };
    if (!kGroup) free_tmem();  // one head: TMEM is no longer needed

    // classification on the certified list
    bool overflow = pending;
    uint32_t keep = 0u, bandm = 0u;
    int need = 0, nb = 0;
    if (!overflow) {
        if (m <= K) {
            keep = alive;  // every candidate; nothing outside can compete
        } else {
            const float lo_cut = __fsub_rd(sK, emax);
            const float hi_cut = __fadd_ru(sK1, emax);
            for (int j = 0; j < m; ++j) {
                const float s = ls[j * kQM + tid];
                const float e = kGroup ? emax : fmaf(eq, kn_s[lc[j * kQM + tid]], fabsf(s) * 0x1p-22f);
                if (__fsub_rd(s, e) > hi_cut) keep |= 1u << j;
                else if (__fadd_ru(s, e) >= lo_cut) bandm |= 1u << j;
            }
            need = K - __popc(keep);
            nb = __popc(bandm);
            if (need >= nb) {
                keep |= bandm;
                need = 0;
            } else if (need > 0) {
                if (nb > kBandCap) {
                    overflow = true;
                } else {
                    const int w0 = atomicAdd(&misc->nwork, nb);
                    uint32_t bm = bandm;
                    for (int k = 0; k < nb; ++k) {
                        const int j = __ffs(bm) - 1;
                        bm &= bm - 1u;
                        bj_s[k * kQM + tid] = (uint8_t)j;
                        work[w0 + k] = (uint16_t)(tid << 3 | k);
                    }
                }
            }
        }
    }
    if (overflow) misc->ovf[atomicAdd(&misc->novf, 1)] = (uint8_t)tid;
    __syncthreads();

    // float64 scores of the band entries, spread over the CTA (grouped heads: the
    // largest of the heads' scores)
    const int nwork = misc->nwork;
    const int64_t qbase = (int64_t)blockIdx.y * a.Lq + i0;  // the CTA's first unit (query, or group query)
    for (int w = tid; w < nwork; w += kTcThreads) {
        const int row = work[w] >> 3, k = work[w] & 7;
        const int c = lc[bj_s[k * kQM + row] * kQM + row];
        double x = -INFINITY;
        int tq;
        QueryCtx q;
        GroupCtx gq;
        if (kGroup) {
            int bb, gg, ii;
            gq = make_group_ctx<bf16, kHD>(a, qbase + row, tq, bb, gg, ii);
        } else {
            q = make_ctx<bf16, kHD>(a, qbase + row, tq);
        }
        for (int hh = 0; hh < G; ++hh) {
            if (kGroup) q = head_ctx(gq, hh, (int)sizeof(bf16));
            const double xh =
                products_exact_f32(qmag_s[hh * kQM + row], kmag_s[hh * ncpad + c])
                    ? exact_score_f32prod(static_cast<const bf16 *>(q.qrow),
                                          static_cast<const bf16 *>(q.khead) + (int64_t)c * q.kst, sc, q.bhead[c])
                    : exact_score<bf16, kHD>(q, c);
            x = fmax(x, xh);
        }
        bx[k * kQM + row] = x;
    }
    __syncthreads();

    // the band's best `need` by (float64 score desc, chunk asc), then the output row
    const bool write_row = !overflow && row_ok;
    if (write_row) {
        if (need > 0) {
            uint32_t taken = 0;
            for (int r = 0; r < need; ++r) {
                double best = -INFINITY;
                int bk = -1, bc = INT_MAX;
                for (int k = 0; k < nb; ++k) {
                    if (taken >> k & 1u) continue;
                    const double x = bx[k * kQM + tid];
                    const int c = lc[bj_s[k * kQM + tid] * kQM + tid];
                    if (bk < 0 || x > best || (x == best && c < bc)) {
                        best = x;
                        bk = k;
                        bc = c;
                    }
                }
                taken |= 1u << bk;
                keep |= 1u << bj_s[bk * kQM + tid];
            }
        }
        const int64_t qi = qbase + tid;
        int32_t *orow = a.idx + qi * K;
        float *srow = a.score + qi * K;
        int o = 0;
        for (int j = 0; j < m; ++j) {
            if (keep >> j & 1u) {
                orow[o] = lc[j * kQM + tid];
                if (!kGroup) srow[o] = ls[j * kQM + tid];
                ++o;
            }
        }
        a.nsel[qi] = o;
        for (; o < K; ++o) {
            orow[o] = -1;
            if (!kGroup) srow[o] = -INFINITY;
        }
    }
    if constexpr (kGroup) {
        // each head's own screen value of the kept chunks, read back from its columns
        // (every lane takes part in the warp-collective loads)
        const int mk = write_row ? m : 0;
        int jj = 0, obase = 0;
        for (int bi = 0; bi < nbat; ++bi) {
            uint32_t msk = 0u;  // kept chunks of this 32-chunk batch (the list ascends)
            for (; jj < mk && lc[jj * kQM + tid] < (bi + 1) * 32; ++jj)
                if (keep >> jj & 1u) msk |= 1u << (lc[jj * kQM + tid] - bi * 32);
            for (int hh = 0; hh < G; ++hh) {
                uint32_t r[32];
                tmem_ld32(trow + hh * args.hcols + bi * 32, r);
                tmem_wait_ld();
                if (msk == 0u) continue;
                float *srow = a.score + (((int64_t)b * a.H + h0 + hh) * a.Lq + i) * K;
                const float *bh = bias_s + hh * ncpad + bi * 32;
                int o = obase;
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    if (msk >> j & 1u) srow[o++] = fmaf(__uint_as_float(r[j]), sc, bh[j]);
            }
            obase += __popc(msk);
        }
        if (write_row)
            for (int hh = 0; hh < G; ++hh) {
                float *srow = a.score + (((int64_t)b * a.H + h0 + hh) * a.Lq + i) * K;
                for (int o = obase; o < K; ++o) srow[o] = -INFINITY;
            }
        free_tmem();
    }

    // rows beyond the list capacity: the exact warp routine, one row per warp
    const int novf = misc->novf;
    if (novf > 0) {
        EntryList &list = *reinterpret_cast<EntryList *>(smem + kFbList + warp * kListBytes);
        for (int r = warp; r < novf; r += kTcThreads / 32) {
            const int row = misc->ovf[r];
            int tq;
            if constexpr (kGroup) {
                float *qs = reinterpret_cast<float *>(smem + kFbQG) + warp * kMaxGroup * kHD;
                int bb, gg, ii;
                const GroupCtx q = make_group_ctx<bf16, kHD>(a, qbase + row, tq, bb, gg, ii);
                for (int hh = 0; hh < G; ++hh) load_query_f32<bf16, kHD>(head_ctx(q, hh, (int)sizeof(bf16)), qs + hh * kHD);
                __syncwarp();
                warp_scan<bf16, kHD>(q, qs, 0, eligible(tq, a.C, a.excl_w), K, list);
                group_write<bf16, kHD>(q, qs, list, a, qbase + row, bb, gg, ii);
            } else {
                float *qs = reinterpret_cast<float *>(smem + kFbQ) + warp * kHD;
                const QueryCtx q = make_ctx<bf16, kHD>(a, qbase + row, tq);
                load_query_f32<bf16, kHD>(q, qs);
                __syncwarp();
                warp_scan<bf16, kHD>(q, qs, 0, eligible(tq, a.C, a.excl_w), K, list);
                warp_write(list, K, qbase + row, a.idx, a.score, a.nsel);
            }
            __syncwarp();
        }
    }
}

constexpr int kMaxSmem = 227 * 1024;  // the opt-in limit; each launch asks for what it uses

}  // namespace

// TMEM columns per head for a CTA whose queries see at most nc chunks.
static uint32_t head_cols(int nc) {
    const int ncpad = (nc + 63) & ~63;
    uint32_t hc = 64;
    while ((int)hc < ncpad) hc <<= 1;
    return hc;
}

bool select_tc_supported(hils_dtype dt, int d, int B, int H, int Lq, int C, int K, bool has_qpos, int G) {
    if (dt != HILS_BF16 || d != kHD || K < 1 || K > kCap - 4) return false;
    if (C < 1 || Lq < 1 || G < 1 || G > kMaxGroup || (int64_t)B * (H / G) > 65535) return false;
    // every query's eligible count, times the heads, fits the TMEM columns; with
    // explicit positions that is only known for C itself
    const int nc = has_qpos ? C : min(C, (Lq - 1) / kChunk);
    if (nc < 1 || C >= 65536) return false;
    const int ncpad = (nc + 63) & ~63;
    if ((int64_t)G * head_cols(nc) > kMaxCols) return false;
    return layout(ncpad, G).total + 1024 <= 227 * 1024;
}

hils_status launch_select_tc(const SelectArgs &a, cudaStream_t s) {
    const int G = a.G;
    const int nc = a.qpos ? a.C : min(a.C, (a.Lq - 1) / kChunk);
    const int ncpad = (nc + 63) & ~63;
    const uint32_t hcols = head_cols(nc);
    uint32_t cols = 32;
    while (cols < (uint32_t)G * hcols) cols <<= 1;
    CUtensorMap mq, mk;
    if (!make_map(&mq, a.Qcal, a.B, a.H, a.Lq, kQM) || !make_map(&mk, a.Ksum, a.B, a.H, a.C, 64))
        return HILS_ERR_CUDA;
    const void *fn = G > 1 ? (const void *)select_tc_kernel<true> : (const void *)select_tc_kernel<false>;
    static KernelSetup setup1, setupg;
    hils_status st = kernel_setup(G > 1 ? setupg : setup1, fn, kTcThreads, kMaxSmem, nullptr);
    if (st != HILS_OK) return st;
    int smem = 1024 + layout(ncpad, G).total;
    // at most 512 / cols CTAs per SM may be resident, so that a TMEM allocation never
    // waits on another CTA: 228 KB of shared memory per SM shared by at most that many
    const int max_ctas = 512 / (int)cols;
    if (max_ctas < 16) smem = max(smem, 233472 / (max_ctas + 1) + 1);
    TcSelArgs ta;
    ta.a = a;
    ta.ncpad = ncpad;
    ta.hcols = hcols;
    ta.cols = cols;
    ta.status = static_cast<uint32_t *>(a.ws);
    dim3 grid((a.Lq + kQM - 1) / kQM, a.B * (a.H / G));
    if (G > 1) select_tc_kernel<true><<<grid, kTcThreads, smem, s>>>(mq, mk, ta);
    else select_tc_kernel<false><<<grid, kTcThreads, smem, s>>>(mq, mk, ta);
    return record_cuda_error(cudaGetLastError());
}

}  // namespace hils
