// The streaming kernels of one PowerSGD step (grouped over all layers).
//
//   pass A: M_w = G_w + E_w (stored over E_w), partial P = sum_w M_w Q per
//           (row, column chunk); the last CTA of a row block sums the chunk
//           partials into P_bar and a float64 Gram partial; the last row
//           block of a layer factors the Gram matrix (Cholesky QR) into T.
//   pass B: P_hat = P_bar T for the tile's rows; partial Q = sum_w M_w^T P_hat
//           per (row block, column); the last CTA of a column chunk sums the
//           row-block partials into Q_bar.
//   pass C: rec = P_hat Q_bar^T per element; E'_w = M_w - rec, optional
//           G_hat = rec, optional momentum.
//
// Step order from "anthology-of-the-sota" note-152 on PowerSGD, "Method".
// At ranks 16 and 32 the two products of passes A and B run on the tf32
// tensor cores (mma.sync, hi/lo-split factors); pass C and every other
// rank use the CUDA cores.  Every cross-CTA sum runs in a fixed order, so
// results are bitwise reproducible.  No CTA waits on another: the last CTA
// to arrive at a counter does the reduction.
#pragma once

#include "device_common.cuh"

namespace psgd {

// ---------------------------------------------------------------------------
// tile decode
struct TileCoord {
    int l, rb, c;
};

// The Q pass (REVERSE) walks the tiles backwards, the other passes
// forwards, so that each pass starts on the tiles the previous one touched
// last, whose lines are still in L2.  The direction is a template argument:
// a run-time select costs the first pass registers it does not have.
template <bool REVERSE>
__device__ __forceinline__ int tile_index() {
    if constexpr (REVERSE) return static_cast<int>(gridDim.x - 1 - blockIdx.x);
    else return static_cast<int>(blockIdx.x);
}

__device__ __forceinline__ TileCoord decode_tile(const LayerDesc& d, int t, int l) {
    const int local = static_cast<int>(t - d.tile_begin);
    TileCoord tc;
    tc.l = l;
    tc.rb = local / d.nchunk;
    tc.c = local - tc.rb * d.nchunk;
    return tc;
}

// ---------------------------------------------------------------------------
// orthogonalisation: factor the r x r Gram matrix (float64) with one warp.
// Cholesky G = R^T R column by column; column j is dropped (row j of R and
// column j of T set to zero) if its pivot, the squared norm of p_bar_j after
// projection on the kept columns before it, is <= drop_tol * max_k G_kk.
// T = R^-1 on the kept columns, so P_hat = P_bar T.
template <int R>
__device__ void factor_gram_warp(const double* Gs, double* Rs, double* Ts, int* drop, int r, double drop_tol,
                                 int lane) {
    for (int idx = lane; idx < R * R; idx += 32) {
        Rs[idx] = 0.0;
        Ts[idx] = 0.0;
    }
    __syncwarp();
    double maxd = 0.0;
    for (int k = 0; k < r; ++k) maxd = fmax(maxd, Gs[k * R + k]);
    const double tau = drop_tol * maxd;
    for (int j = 0; j < r; ++j) {
        double d = Gs[j * R + j];
        for (int k = 0; k < j; ++k) d -= Rs[k * R + j] * Rs[k * R + j];
        const bool dropped = (d <= tau);
        const double rjj = dropped ? 0.0 : sqrt(d);
        const int i = lane;
        if (i > j && i < r) {
            double s = Gs[j * R + i];
            for (int k = 0; k < j; ++k) s -= Rs[k * R + j] * Rs[k * R + i];
            Rs[j * R + i] = dropped ? 0.0 : s / rjj;
        }
        __syncwarp();
        if (lane == 0) {
            Rs[j * R + j] = rjj;
            drop[j] = dropped ? 1 : 0;
        }
        __syncwarp();
    }
    for (int j = 0; j < r; ++j) {
        const int l = lane;
        if (l <= j) {
            double t;
            if (drop[j]) {
                t = 0.0;
            } else if (l == j) {
                t = 1.0 / Rs[j * R + j];
            } else {
                double s = 0.0;
                for (int k = l; k < j; ++k) s += Ts[l * R + k] * Rs[k * R + j];
                t = -s / Rs[j * R + j];
            }
            Ts[l * R + j] = t;
        }
        __syncwarp();
    }
}

// ---------------------------------------------------------------------------
// pass A

// Ranks 16 and 32 use the wide kernels: a chunk (up to 32 * VEC columns) is
// walked in sub-chunks of 32 columns.  Passes A and B form M * Q and
// P_hat^T * M on the tensor cores (mma.sync m16n8k8 tf32, a warp per 16
// rows); pass C forms the reconstruction once per tile on the CUDA cores
// and applies it to every worker.  Tiles of the wide kernels have 16, 32 or
// 64 rows.
template <int R>
struct IsWide { static constexpr bool value = R >= 16; };   // pass C: the wide variant
template <int R>
struct UseMma { static constexpr bool value = R >= 16; };   // passes A and B: tensor cores
constexpr int kWideCols = 32;
constexpr int kWideRows = 64;    // rows per tile cap for the wide kernels

// ---- float32 products on the tf32 tensor cores ---------------------------
// x = hi + lo with hi = x rounded to tf32 (10 mantissa bits, to nearest,
// ties away) and lo = (x - hi) rounded to tf32; x - hi is exact.  A product
// a * b is taken as a_hi b_hi + a_hi b_lo + a_lo b_hi: the dropped a_lo b_lo
// and the rounding of the lo parts leave a relative error below 2^-21
// (split-precision products on tensor cores: Markidis et al., "NVIDIA
// Tensor Core Programmability, Performance & Precision", IPDPSW 2018).
// Rounding to tf32 on the bit pattern: the magnitude bits plus half a unit of
// the 13 dropped bits, then truncated.  IEEE sign-magnitude encoding makes
// this round-to-nearest with ties away from zero (a carry out of the
// mantissa moves to the next binade; infinity stays infinity), computed on
// the integer pipe instead of the conversion unit.  Any rounding to tf32
// would do: hi + lo = x holds exactly whichever way hi is rounded.
// The first pass is bound by the conversion unit (its float64 flushes), so
// it rounds on the integer pipe; the second pass, whose conversion unit is
// idle and whose registers are at their limit, uses cvt.rna.tf32.f32.
__device__ __forceinline__ uint32_t tf32_round_int(float x) {
    return (__float_as_uint(x) + 0x1000u) & 0xffffe000u;
}
__device__ __forceinline__ uint32_t tf32_round(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}
// sum_{j < count} src[j * stride] in index order, eight loads in flight at a
// time (the partials were written by other CTAs of this launch: L2 loads)
__device__ __forceinline__ double sum_in_order(const double* src, int64_t stride, int count) {
    double s = 0.0;
    int j = 0;
    for (; j + 8 <= count; j += 8) {
        double v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) v[u] = __ldcg(src + (j + u) * stride);
#pragma unroll
        for (int u = 0; u < 8; ++u) s += v[u];
    }
    for (; j < count; ++j) s += __ldcg(src + j * stride);
    return s;
}

// elements summed together by sums_in_order: four at ranks 16 and 32, two
// below (those kernels run at 80 registers per thread)
template <int R>
struct SumBatch { static constexpr int value = R >= 16 ? 4 : 2; };

// s[e] = sum_{j < count} src[e][j * stride] for E elements at once, each in
// index order (the same order as sum_in_order), eight loads per element in
// flight; elements with valid[e] false read nothing and their s[e] is 0
template <int E>
__device__ __forceinline__ void sums_in_order(const double* const (&src)[E], const bool (&valid)[E],
                                              int64_t stride, int count, double (&s)[E]) {
#pragma unroll
    for (int e = 0; e < E; ++e) s[e] = 0.0;
    int j = 0;
    for (; j + 8 <= count; j += 8) {
        double v[E][8];
#pragma unroll
        for (int e = 0; e < E; ++e)
#pragma unroll
            for (int u = 0; u < 8; ++u) v[e][u] = valid[e] ? __ldcg(src[e] + (j + u) * stride) : 0.0;
#pragma unroll
        for (int e = 0; e < E; ++e)
#pragma unroll
            for (int u = 0; u < 8; ++u) s[e] += v[e][u];
    }
    for (; j < count; ++j)
#pragma unroll
        for (int e = 0; e < E; ++e)
            if (valid[e]) s[e] += __ldcg(src[e] + j * stride);
}
__device__ __forceinline__ void tf32_split(float x, uint32_t& hi, uint32_t& lo) {
    hi = tf32_round(x);
    lo = tf32_round(x - __uint_as_float(hi));
}
__device__ __forceinline__ void tf32_split_int(float x, uint32_t& hi, uint32_t& lo) {
    hi = tf32_round_int(x);
    lo = tf32_round_int(x - __uint_as_float(hi));
}
// c += A (16 x 8, row-major fragment) * B (8 x 8, column fragment), float32
// accumulate.  Fragment of lane (g = lane / 4, t = lane % 4): a = A[g][t],
// A[g + 8][t], A[g][t + 4], A[g + 8][t + 4]; b = B[t][g], B[t + 4][g];
// c = C[g][2t], C[g][2t + 1], C[g + 8][2t], C[g + 8][2t + 1].
__device__ __forceinline__ void mma_tf32(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// 3-term split product of one k-step: c = A B (c starts at zero)
__device__ __forceinline__ void mma_tf32x3(float (&c)[4], const uint32_t (&ahi)[4], const uint32_t (&alo)[4],
                                           const float4& b) {
    // b = (b0 hi, b1 hi, b0 lo, b1 lo); small terms first
    mma_tf32(c, alo, __float_as_uint(b.x), __float_as_uint(b.y));
    mma_tf32(c, ahi, __float_as_uint(b.z), __float_as_uint(b.w));
    mma_tf32(c, ahi, __float_as_uint(b.x), __float_as_uint(b.y));
}

// ---- asynchronous global -> shared copies (16 bytes, no register staging) --
// cp.async with a source size of 0 writes zeros (used for rows and columns
// outside the layer; the source address is then never read).
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc, bool valid) {
    const unsigned dst = static_cast<unsigned>(__cvta_generic_to_shared(smem_dst));
    const int n = valid ? 16 : 0;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(gsrc), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory"); }

// ---- 5th-generation tensor cores (tcgen05) --------------------------------
// Shared-memory matrix descriptor, no swizzle, K-major operand: core
// matrices of 8 rows (of M or N) x 16 bytes (4 tf32 of K) stored as 128
// contiguous bytes; LBO is the byte distance between core matrices adjacent
// in K, SBO between core matrices adjacent in M or N.  Field layout of the
// sm_100 matrix descriptor: start address >> 4 in bits [0, 14), LBO >> 4 in
// [16, 30), SBO >> 4 in [32, 46), descriptor version 1 in [46, 48), base
// offset 0, layout type 0 (no swizzle) in [61, 64).
__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    return static_cast<uint64_t>((saddr >> 4) & 0x3fffu) | (static_cast<uint64_t>((lbo >> 4) & 0x3fffu) << 16) |
           (static_cast<uint64_t>((sbo >> 4) & 0x3fffu) << 32) | (1ull << 46);
}
// Instruction descriptor of kind::tf32 with both operands K-major: D
// float32 (bits [4, 6) = 1), A and B tf32 (bits [7, 10), [10, 13) = 2),
// N >> 3 in bits [17, 23), M >> 4 in bits [24, 29).  (Operands marked
// MN-major in bits 15 and 16 were measured to contribute nothing to D for
// tf32 on this part; the kernels transpose into K-major instead.)
__host__ __device__ constexpr uint32_t umma_idesc_tf32(int M, int N) {
    return (1u << 4) | (2u << 7) | (2u << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
           (static_cast<uint32_t>(M >> 4) << 24);
}
__device__ __forceinline__ void umma_tf32(uint32_t tmem_d, uint64_t da, uint64_t db, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}\n" ::"r"(tmem_d),
        "l"(da), "l"(db), "r"(idesc), "r"(acc), "r"(0u), "r"(0u), "r"(0u), "r"(0u));
}
// The same with A read from tensor memory (K-major: lane = row of M, one
// column per tf32 element of K) at tmem_a.
__device__ __forceinline__ void umma_tf32_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t db, uint32_t idesc,
                                             uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], [%1], %2, %3, {%5, %6, %7, %8}, p;\n\t}\n" ::"r"(tmem_d),
        "r"(tmem_a), "l"(db), "r"(idesc), "r"(acc), "r"(0u), "r"(0u), "r"(0u), "r"(0u));
}
// 16 consecutive columns of this thread's TMEM lane (the warp's 32 lanes)
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&u)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15, %16};" ::"r"(taddr),
        "r"(u[0]), "r"(u[1]), "r"(u[2]), "r"(u[3]), "r"(u[4]), "r"(u[5]), "r"(u[6]), "r"(u[7]), "r"(u[8]),
        "r"(u[9]), "r"(u[10]), "r"(u[11]), "r"(u[12]), "r"(u[13]), "r"(u[14]), "r"(u[15])
        : "memory");
}
// 8 consecutive columns of this thread's TMEM lane (the warp's 32 lanes)
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&u)[8]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
                 "r"(u[0]), "r"(u[1]), "r"(u[2]), "r"(u[3]), "r"(u[4]), "r"(u[5]), "r"(u[6]), "r"(u[7])
                 : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
// one lane of the (converged) warp: true there, false elsewhere
__device__ __forceinline__ bool elect_one() {
    uint32_t pred;
    asm volatile(
        "{\n\t.reg .pred P;\n\telect.sync _|P, 0xffffffff;\n\tselp.b32 %0, 1, 0, P;\n\t}\n"
        : "=r"(pred));
    return pred != 0;
}
__device__ __forceinline__ void umma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
// Bounded wait for the phase `parity` of an mbarrier to complete: about one
// second at most, after which the status word gets kStatusTimeout and false
// is returned (the caller then winds down without using the results).
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity, int* status) {
    const uint64_t t0 = global_timer_ns();
    for (;;) {
        uint32_t ok;
        asm volatile(
            "{\n\t.reg .pred P1;\n\tmbarrier.try_wait.parity.shared::cta.b64 P1, [%1], %2;\n\t"
            "selp.b32 %0, 1, 0, P1;\n\t}\n"
            : "=r"(ok)
            : "r"(bar), "r"(parity)
            : "memory");
        if (ok) return true;
        if (global_timer_ns() - t0 > 1000000000ull) {
            atomicOr(status, kStatusTimeout);
            return false;
        }
    }
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// Staged second pass (ranks 16, 32; rows 16-byte aligned, i.e. n % 4 == 0):
// one worker's 64 x 128 block of M at a time goes to shared memory by
// cp.async (kStages buffers), row stride kStgStride floats (the padding
// keeps a quarter-warp's 8-byte fragment loads on distinct banks).
constexpr int kStgRows = 64;
constexpr int kStgCols = 128;
constexpr int kStgStride = kStgCols + 8;
constexpr int kStages = 2;
constexpr size_t kStgBytes = static_cast<size_t>(kStages) * kStgRows * kStgStride * sizeof(float);
// Tensor-core second pass: B = [P_hat hi | P_hat lo] K-major in shared
// memory (8 rows of N x 16 bytes per core matrix, 16 core matrices = 64
// rows of K per group of 8 N rows), the threads' float64 sums, then the
// mbarrier, the TMEM address and the wind-down flag.  A (the worker's block split into hi and lo) and the
// accumulators live in tensor memory.
constexpr uint32_t kTcSboB = 16 * 128;
// workers whose products accumulate in tensor memory (float32, at most 64
// MMA accumulations per element and half) before D is read back into the
// float64 sums
constexpr int kTcGroup = 4;
// independent accumulators (k-step ks goes to ks % kTcChains)
constexpr int kTcChains = 2;
// tensor-memory columns: A hi (64 rows of K), A lo, then the chains' D
constexpr uint32_t kTcAHi = 0, kTcALo = 64, kTcD = 128;
template <int R>
struct TcSmem {
    static constexpr size_t b_bytes = static_cast<size_t>(2 * R / 8) * kTcSboB;   // 2R rows of N x 64 of K
    // each thread's float64 sums of its column and rank half: [R / 2][threads]
    static constexpr size_t sum_bytes = static_cast<size_t>(R / 2) * kThreads * sizeof(double);
    // at least 76 KB, so that no more than two CTAs reside on an SM (228 KB)
    // and their tensor memory (tmem_cols each) fits in the SM's 512 columns
    static constexpr size_t need = b_bytes + sum_bytes + 16;
    static constexpr size_t total = need > 76 * 1024 ? need : 76 * 1024;
    // per chain D = [hi*hi + lo*hi | hi*lo]; the allocation is a power of two
    static constexpr uint32_t tmem_cols = 256;
    static_assert(kTcD + kTcChains * 2 * R <= tmem_cols, "tensor memory of the second pass");
};

constexpr int kMmaRows = 16;                  // rows per warp in the tensor-core pass A
constexpr int kMaxKSteps = 32 * 4 / 8;        // k-steps of 8 columns in the widest chunk
constexpr size_t kQfBytes = static_cast<size_t>(kMaxKSteps) * 4 * 32 * sizeof(float4);
constexpr int kRedStride = 32 + 1;            // second pass: warp partial row stride (floats)
constexpr size_t kPaBytes = static_cast<size_t>(kWarps) * 2 * 2 * 32 * 8 * sizeof(float);   // its A fragments
constexpr int kRecStride = 4 * kWideCols + 1;  // lazy reconstruction tile row stride (floats)
constexpr size_t kRecBytes = static_cast<size_t>(kWideRows) * kRecStride * sizeof(float);

template <int R>
struct SmemA {
    // layout inside dynamic shared memory (bytes)
    static __host__ __device__ size_t ptr_bytes(int W) { return static_cast<size_t>(2 * W) * sizeof(void*); }
    static __host__ __device__ size_t rows_bytes(int tm) { return static_cast<size_t>(tm) * R * sizeof(double); }
    static __host__ __device__ size_t fac_bytes() { return 3 * R * R * sizeof(double) + 2 * R * sizeof(int) + 64; }
    // tensor-core kernel: the chunk's split Q fragments (later the parts'
    // P partials, kWarps x 16 x 32 doubles, the same 32 KB) and, in the
    // lazy representation, the tile's reconstruction
    static __host__ __device__ size_t wide_bytes(bool lazy) {
        return UseMma<R>::value ? kQfBytes + (lazy ? kRecBytes : 0) : 0;
    }
    static __host__ __device__ size_t total(int W, int tm, bool lazy) {
        return ((ptr_bytes(W) + 15) & ~size_t(15)) + ((rows_bytes(tm) + 15) & ~size_t(15)) +
               ((fac_bytes() + 15) & ~size_t(15)) + wide_bytes(lazy);
    }
};

template <int R, int VEC, typename GT, bool LAZY, bool SF, bool READM>
__device__ __forceinline__ void pass_a_rows(const Params& p, const LayerDesc& d, const TileCoord& tc,
                                            const GT* const* gp, float* const* ep, const float* ph_prev) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int r = p.r;
    const int W = p.workers;
    const int64_t n = d.n, m = d.m;
    const int64_t i0 = static_cast<int64_t>(tc.rb) * d.tm;
    const int64_t i1 = min(i0 + d.tm, m);
    const int s0 = tc.c * d.slots;
    const int ns = min(d.slots, d.nvec - s0);
    const bool active = lane < ns;
    const int64_t j = static_cast<int64_t>(s0 + (active ? lane : 0)) * VEC;

    // warm-start Q rows of this lane's columns, zero-padded to R
    float qv[VEC][R];
    {
        const float* Q = p.t.q[tc.l];
#pragma unroll
        for (int v = 0; v < VEC; ++v)
#pragma unroll
            for (int k = 0; k < R; ++k) qv[v][k] = (active && k < r) ? Q[(j + v) * r + k] : 0.f;
    }
    // previous Q_bar for rebuilding E' (lazy representation)
    float qp[LAZY ? VEC : 1][LAZY ? R : 1];
    if constexpr (LAZY) {
        const float* Qb = p.ws.qbar + d.qrow_off;
#pragma unroll
        for (int v = 0; v < VEC; ++v)
#pragma unroll
            for (int k = 0; k < R; ++k) qp[v][k] = (active && p.use_prev) ? Qb[(j + v) * R + k] : 0.f;
    }

    double* ppart = p.ws.ppart + d.ppart_off;
    constexpr int U = (VEC == 4) ? 4 : 8;
    // products are summed in float32 over runs of 8 terms (F workers x VEC
    // columns), then added to the float64 row accumulator
    constexpr int F = 8 / VEC;
    static_assert(U % F == 0, "flush interval must divide the unroll");
    constexpr int LG = Log2<R>::value;

    for (int64_t i = i0 + warp; i < i1; i += kWarps) {
        double acc[R];
#pragma unroll
        for (int k = 0; k < R; ++k) acc[k] = 0.0;
        if (active) {
            const int64_t base = i * n + j;
            float rec[VEC];
            if constexpr (LAZY) {
                float ph[R];
#pragma unroll
                for (int k = 0; k < R; ++k) ph[k] = ph_prev[(i - i0) * R + k];
#pragma unroll
                for (int v = 0; v < VEC; ++v) rec[v] = recon_dot<R>(ph, qp[v]);
            }
            float msum[VEC];
#pragma unroll
            for (int v = 0; v < VEC; ++v) msum[v] = 0.f;
            // G workers' loads in flight, then M, the store and the products;
            // float32 runs are flushed every F workers (<= 8 terms)
            auto group = [&](auto GC, int w0) {
                constexpr int G = decltype(GC)::value;
                [[maybe_unused]] float g[G][VEC];
                float e[G][VEC];
#pragma unroll
                for (int u = 0; u < G; ++u) {
                    if constexpr (!READM) ld_grad<GT, VEC>(gp[w0 + u] + base, g[u]);
                    ld_f32<VEC>(ep[w0 + u] + base, e[u]);
                }
                if constexpr (!READM) {
#pragma unroll
                    for (int u = 0; u < G; ++u) {
#pragma unroll
                        for (int v = 0; v < VEC; ++v) {
                            float ev = e[u][v];
                            if constexpr (LAZY) ev = ev - rec[v];
                            e[u][v] = g[u][v] + ev;
                        }
                        st_f32<VEC>(ep[w0 + u] + base, e[u]);
                    }
                }
                if constexpr (SF) {
#pragma unroll
                    for (int u = 0; u < G; ++u)
#pragma unroll
                        for (int v = 0; v < VEC; ++v) msum[v] += e[u][v];
                } else {
                    float pw[R];
#pragma unroll
                    for (int k = 0; k < R; ++k) pw[k] = 0.f;
#pragma unroll
                    for (int u = 0; u < G; ++u) {
#pragma unroll
                        for (int v = 0; v < VEC; ++v) axpy<R>(pw, e[u][v], qv[v]);
                        if ((u + 1) % F == 0 || u + 1 == G) {
#pragma unroll
                            for (int k = 0; k < R; ++k) {
                                acc[k] += static_cast<double>(pw[k]);
                                pw[k] = 0.f;
                            }
                        }
                    }
                }
            };
            int w = 0;
            for (; w + U <= W; w += U) group(std::integral_constant<int, U>{}, w);
            if constexpr (U > 4) {
                if (w + 4 <= W) {
                    group(std::integral_constant<int, 4>{}, w);
                    w += 4;
                }
            }
            if constexpr (U > 2) {
                if (w + 2 <= W) {
                    group(std::integral_constant<int, 2>{}, w);
                    w += 2;
                }
            }
            if (w < W) group(std::integral_constant<int, 1>{}, w);
            if constexpr (SF) {
                float pw[R];
#pragma unroll
                for (int k = 0; k < R; ++k) pw[k] = 0.f;
#pragma unroll
                for (int v = 0; v < VEC; ++v)
                    axpy<R>(pw, msum[v], qv[v]);
#pragma unroll
                for (int k = 0; k < R; ++k) acc[k] = static_cast<double>(pw[k]);
            }
        }
        TransposeReduce<double, R, 16>::run(acc, lane);
        if ((lane & ((32 >> LG) - 1)) == 0) {
            const int k = lane >> (5 - LG);
            ppart[(static_cast<int64_t>(tc.c) * m + i) * R + k] = acc[0];
        }
    }
}

// Tensor-core variant of the first pass (R = 32).  The tile's rows split
// into row groups of 16 (tm / 16 of them); each row group belongs to
// kWarps / (tm / 16) warps ("parts") that deal the workers among
// themselves.  For every (sub-chunk of 32 columns, worker) of its share a
// warp loads G and E of its 16 x 32 block straight into the registers of
// the mma A fragments (VEC-wide loads), forms M = G + E there, stores M
// over E, prefetches the next block and multiplies: per k-step of 8
// columns and 8 ranks, three tf32 products (mma_tf32x3) summed in float32,
// then added to a Kahan-compensated float32 accumulator, which is widened to
// float64 at the end of the tile.  The parts' partials are then added in
// part order (float64) and written per chunk.
//
// Fragment columns.  An mma k-step takes 8 columns in any order, as long
// as A and B agree.  Lane (g, t) holds rows g and g + 8 and, in k-step ks,
// the columns col0(ks) (slot t) and col1(ks) (slot t + 4) of the sub-chunk:
//   VEC 4: col0 = 16 (ks / 2) + 4 t + 2 (ks % 2), col1 = col0 + 1
//   VEC 2: col0 = 8 ks + 2 t,                   col1 = col0 + 1
//   VEC 1: col0 = 8 ks + t,                     col1 = col0 + 4
// so a VEC-wide load of one row fills slots of one or two k-steps.
template <int VEC>
__device__ __forceinline__ int frag_col0(int ks, int t4) {
    if constexpr (VEC == 4) return 16 * (ks >> 1) + 4 * t4 + 2 * (ks & 1);
    else if constexpr (VEC == 2) return 8 * ks + 2 * t4;
    else return 8 * ks + t4;
}
template <int VEC>
__device__ __forceinline__ int frag_col1(int ks, int t4) {
    return frag_col0<VEC>(ks, t4) + (VEC == 1 ? 4 : 1);
}

// G or E block of one (sub-chunk, worker) into fragment order:
// v[ks][0] = (row g, col0), v[ks][1] = (row g + 8, col0),
// v[ks][2] = (row g, col1), v[ks][3] = (row g + 8, col1); zero outside the
// layer.  base points at (tile row r0, sub-chunk column 0) of the buffer.
template <int VEC, typename T>
__device__ __forceinline__ void load_frag(const T* base, int64_t n, int g, int t4, bool ok_lo, bool ok_hi, int cols,
                                          float (&v)[4][4]) {
#pragma unroll
    for (int ks = 0; ks < 4; ++ks)
#pragma unroll
        for (int q = 0; q < 4; ++q) v[ks][q] = 0.f;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
        const bool ok_row = half ? ok_hi : ok_lo;
        const int q0 = half;   // 0: row g, 1: row g + 8
        const T* rp = base + static_cast<int64_t>(g + 8 * half) * n;
        if constexpr (VEC == 4) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int c = 16 * h + 4 * t4;
                if (ok_row && c < cols) {
                    float x[4];
                    if constexpr (std::is_same<T, float>::value) ld_f32<4>(rp + c, x);
                    else ld_grad<T, 4>(rp + c, x);
                    v[2 * h][q0] = x[0];
                    v[2 * h][q0 + 2] = x[1];
                    v[2 * h + 1][q0] = x[2];
                    v[2 * h + 1][q0 + 2] = x[3];
                }
            }
        } else if constexpr (VEC == 2) {
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                const int c = 8 * ks + 2 * t4;
                if (ok_row && c < cols) {
                    float x[2];
                    if constexpr (std::is_same<T, float>::value) ld_f32<2>(rp + c, x);
                    else ld_grad<T, 2>(rp + c, x);
                    v[ks][q0] = x[0];
                    v[ks][q0 + 2] = x[1];
                }
            }
        } else {
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
#pragma unroll
                for (int s2 = 0; s2 < 2; ++s2) {
                    const int c = 8 * ks + t4 + 4 * s2;
                    if (ok_row && c < cols) {
                        float x[1];
                        if constexpr (std::is_same<T, float>::value) ld_f32<1>(rp + c, x);
                        else ld_grad<T, 1>(rp + c, x);
                        v[ks][q0 + 2 * s2] = x[0];
                    }
                }
            }
        }
    }
}

// M block (fragment order) stored back over E, same addressing as load_frag.
template <int VEC>
__device__ __forceinline__ void store_frag(float* base, int64_t n, int g, int t4, bool ok_lo, bool ok_hi, int cols,
                                           const float (&v)[4][4]) {
#pragma unroll
    for (int half = 0; half < 2; ++half) {
        const bool ok_row = half ? ok_hi : ok_lo;
        const int q0 = half;
        float* rp = base + static_cast<int64_t>(g + 8 * half) * n;
        if constexpr (VEC == 4) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int c = 16 * h + 4 * t4;
                if (ok_row && c < cols) {
                    const float x[4] = {v[2 * h][q0], v[2 * h][q0 + 2], v[2 * h + 1][q0], v[2 * h + 1][q0 + 2]};
                    st_f32<4>(rp + c, x);
                }
            }
        } else if constexpr (VEC == 2) {
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                const int c = 8 * ks + 2 * t4;
                if (ok_row && c < cols) {
                    const float x[2] = {v[ks][q0], v[ks][q0 + 2]};
                    st_f32<2>(rp + c, x);
                }
            }
        } else {
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
#pragma unroll
                for (int s2 = 0; s2 < 2; ++s2) {
                    const int c = 8 * ks + t4 + 4 * s2;
                    if (ok_row && c < cols) rp[c] = v[ks][q0 + 2 * s2];
                }
        }
    }
}

template <int R, int VEC, typename GT, bool LAZY, bool SF, bool READM>
__device__ __forceinline__ void pass_a_mma(const Params& p, const LayerDesc& d, const TileCoord& tc,
                                           const GT* const* gp, float* const* ep, const float* ph_prev,
                                           unsigned char* wide) {
    static_assert(R == 16 || R == 32, "tensor-core pass A: rank 16 or 32");
    constexpr int NT = R / 8;                   // n-tiles of 8 ranks
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, t4 = lane & 3;
    const int r = p.r;
    const int W = p.workers;
    const int64_t n = d.n, m = d.m;
    const int64_t i0 = static_cast<int64_t>(tc.rb) * d.tm;
    const int rows = static_cast<int>(min(static_cast<int64_t>(d.tm), m - i0));
    const int64_t jc = static_cast<int64_t>(tc.c) * d.slots * d.vec;
    const int width = static_cast<int>(min(static_cast<int64_t>(d.slots) * d.vec, n - jc));
    const int nsc = (width + kWideCols - 1) / kWideCols;
    const int nrg = d.tm / kMmaRows;            // 1, 2 or 4 row groups
    const int parts = kWarps / nrg;
    const int rg = warp % nrg, part = warp / nrg;
    const int r0 = rg * kMmaRows;               // first tile row of this warp
    const bool ok_lo = r0 + g < rows, ok_hi = r0 + g + 8 < rows;
    float4* qf = reinterpret_cast<float4*>(wide);   // [k-step][rank tile][lane]

    // split B fragments of the chunk's Q in the same column order (zero
    // beyond the chunk and rank r)
    {
        const float* Q = p.t.q[tc.l];
        const int nks = nsc * 4;
        for (int idx = threadIdx.x; idx < nks * NT * 32; idx += kThreads) {
            const int ln = idx & 31, nt = (idx >> 5) % NT, ksg = (idx >> 5) / NT;
            const int sc = ksg >> 2, ks = ksg & 3;
            const int jj0 = sc * kWideCols + frag_col0<VEC>(ks, ln & 3);
            const int jj1 = sc * kWideCols + frag_col1<VEC>(ks, ln & 3);
            const int k = 8 * nt + (ln >> 2);
            const float b0 = (jj0 < width && k < r) ? Q[(jc + jj0) * r + k] : 0.f;
            const float b1 = (jj1 < width && k < r) ? Q[(jc + jj1) * r + k] : 0.f;
            uint32_t h0, l0, h1, l1;
            tf32_split(b0, h0, l0);
            tf32_split(b1, h1, l1);
            qf[idx] = make_float4(__uint_as_float(h0), __uint_as_float(h1), __uint_as_float(l0), __uint_as_float(l1));
        }
    }
    __syncthreads();

    // this part's workers: part, part + parts, ...
    const int nw = W > part ? (W - part + parts - 1) / parts : 0;
    const int total = nsc * nw;
    const int64_t row0 = (i0 + r0) * n + jc;    // (first row of this warp, chunk column 0)
    float gq[4][4], eq[4][4];
    auto load = [&](int sc, int w) {
        const int cols = width - sc * kWideCols;
        load_frag<VEC>(ep[w] + row0 + sc * kWideCols, n, g, t4, ok_lo, ok_hi, cols, eq);
        if constexpr (!READM) load_frag<VEC>(gp[w] + row0 + sc * kWideCols, n, g, t4, ok_lo, ok_hi, cols, gq);
    };

    // Kahan-compensated float32 sums of the k-steps' products (Kahan 1965):
    // the running sum and its compensation stay on the FMA pipe, accurate
    // to about one float32 rounding of the sum however many k-steps it
    // takes; the tile's result is widened to float64 once, below.
    float accf[NT][4], comp[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int c = 0; c < 4; ++c) accf[nt][c] = comp[nt][c] = 0.f;
    float* rt = reinterpret_cast<float*>(wide + kQfBytes);   // lazy: [tile row][chunk column]
    float msum[SF ? 4 : 1][SF ? 4 : 1];
    if constexpr (LAZY) {
        // the previous step's reconstruction of the whole tile (every row
        // and every column slot, zero beyond the chunk), once, by all
        // threads: recon_dot's operation order per element, two columns
        // per packed FMA
        const float* Qb = p.ws.qbar + d.qrow_off;
        const int c0 = 2 * (threadIdx.x & 63), rq = threadIdx.x >> 6;
        const bool ok0 = c0 < width && p.use_prev, ok1 = c0 + 1 < width && p.use_prev;
        float2 qp[R];
#pragma unroll
        for (int kk = 0; kk < R; ++kk)
            qp[kk] = make_float2(ok0 ? Qb[(jc + c0) * R + kk] : 0.f, ok1 ? Qb[(jc + c0 + 1) * R + kk] : 0.f);
        for (int ii = rq; ii < d.tm; ii += 4) {
            const float* ph = ph_prev + min(ii, rows - 1) * R;
            float2 s2 = make_float2(0.f, 0.f);
#pragma unroll
            for (int kk = 0; kk < R; ++kk) s2 = __ffma2_rn(make_float2(ph[kk], ph[kk]), qp[kk], s2);
            rt[ii * kRecStride + c0] = s2.x;
            rt[ii * kRecStride + c0 + 1] = s2.y;
        }
        __syncthreads();
    }

    // products of an M block (fragment order) with the sub-chunk's k-steps
    auto multiply = [&](int sc, const float (&mv)[4][4]) {
        const int cols = width - sc * kWideCols;
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
            // does k-step ks hold a column of the sub-chunk? (VEC 4: k-steps
            // 2h and 2h + 1 share columns 16h .. 16h + 15)
            if ((VEC == 4 ? 16 * (ks >> 1) : 8 * ks) < cols) {
                uint32_t ahi[4], alo[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) tf32_split_int(mv[ks][q], ahi[q], alo[q]);
                const float4* qk = qf + ((sc * 4 + ks) * NT) * 32 + lane;
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    float c[4] = {0.f, 0.f, 0.f, 0.f};
                    mma_tf32x3(c, ahi, alo, qk[nt * 32]);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const float y = c[q] - comp[nt][q];
                        const float t = accf[nt][q] + y;
                        comp[nt][q] = (t - accf[nt][q]) - y;
                        accf[nt][q] = t;
                    }
                }
            }
        }
    };

    if (total > 0) load(0, part);
    int sc = 0, wi = 0;
    for (int it = 0; it < total; ++it) {
        const int w = part + wi * parts;
        const int cols = width - sc * kWideCols;
        if (wi == 0) {
            if constexpr (SF) {
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
#pragma unroll
                    for (int q = 0; q < 4; ++q) msum[ks][q] = 0.f;
            }
        }
        // M for this worker's block, in the fragment registers
        float mv[4][4];
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                float x = eq[ks][q];
                if constexpr (!READM) {
                    if constexpr (LAZY) {
                        const int c = (q & 2) ? frag_col1<VEC>(ks, t4) : frag_col0<VEC>(ks, t4);
                        x = x - rt[(r0 + g + 8 * (q & 1)) * kRecStride + sc * kWideCols + c];
                    }
                    x = gq[ks][q] + x;
                }
                mv[ks][q] = x;
            }
        if constexpr (!READM) store_frag<VEC>(ep[w] + row0 + sc * kWideCols, n, g, t4, ok_lo, ok_hi, cols, mv);
        const bool last_w = wi == nw - 1;
        // next (sub-chunk, worker) in flight while this block is multiplied
        int sc2 = sc, wi2 = wi + 1;
        if (wi2 == nw) {
            wi2 = 0;
            ++sc2;
        }
        if (it + 1 < total) load(sc2, part + wi2 * parts);
        if constexpr (SF) {
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
#pragma unroll
                for (int q = 0; q < 4; ++q) msum[ks][q] += mv[ks][q];
            if (last_w) multiply(sc, msum);
        } else {
            multiply(sc, mv);
        }
        sc = sc2;
        wi = wi2;
    }

    double acc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[nt][q] = static_cast<double>(accf[nt][q]) - static_cast<double>(comp[nt][q]);

    // parts' partials added in part order; part 0 writes the chunk's rows
    __syncthreads();   // every warp is done with the Q fragments
    double* cb = reinterpret_cast<double*>(wide);   // [warp][4 NT values][lane]
    if (part > 0) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int q = 0; q < 4; ++q) cb[(warp * 4 * NT + nt * 4 + q) * 32 + lane] = acc[nt][q];
    }
    __syncthreads();
    if (part == 0) {
        for (int pp = 1; pp < parts; ++pp) {
            const int src = pp * nrg + rg;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int q = 0; q < 4; ++q) acc[nt][q] += cb[(src * 4 * NT + nt * 4 + q) * 32 + lane];
        }
        double* ppart = p.ws.ppart + d.ppart_off;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int ii = r0 + g + 8 * (q >> 1);
                const int k = 8 * nt + 2 * t4 + (q & 1);
                if (ii < rows) ppart[(static_cast<int64_t>(tc.c) * m + i0 + ii) * R + k] = acc[nt][q];
            }
    }
}

// Last CTA of a row block: P_bar rows and the Gram partial.  Last row block
// of a layer: Gram sum and factorisation.
template <int R>
__device__ void pass_a_epilogue(const Params& p, const LayerDesc& d, const TileCoord& tc, double* pb_s,
                                unsigned char* fac) {
    __shared__ int s_flag;
    constexpr int NG = R * (R + 1) / 2;
    const int tid = threadIdx.x;
    const CounterLayout cl = counter_layout(d.nrb, d.nsup, d.nchunk);
    unsigned* cnt = p.ws.cnt + d.cnt_off;

    // 1) the last chunk tile of a row block: P_bar rows and the Gram partial
    __syncthreads();
    if (tid == 0) {
        __threadfence();
        const unsigned prev = atomicAdd(&cnt[cl.a_rb + tc.rb], 1u);
        if (prev >= static_cast<unsigned>(d.nchunk)) atomicOr(p.ws.status, kStatusCounter);
        s_flag = (prev == static_cast<unsigned>(d.nchunk - 1));
    }
    __syncthreads();
    if (!s_flag) return;
    __threadfence();

    const int64_t m = d.m;
    const int64_t i0 = static_cast<int64_t>(tc.rb) * d.tm;
    const int rows = static_cast<int>(min(static_cast<int64_t>(d.tm), m - i0));
    const double* ppart = p.ws.ppart + d.ppart_off;
    double* pbar = p.ws.pbar + d.prow_off;
    const double inv_w = 1.0 / static_cast<double>(p.workers);
    for (int base = tid; base < rows * R; base += SumBatch<R>::value * kThreads) {
        constexpr int E = SumBatch<R>::value;
        const double* src[E];
        bool valid[E];
        double sums[E];
#pragma unroll
        for (int e = 0; e < E; ++e) {
            const int idx = base + e * kThreads;
            valid[e] = idx < rows * R;
            src[e] = ppart + (i0 + (valid[e] ? idx / R : 0)) * R + (valid[e] ? idx % R : 0);
        }
        sums_in_order<E>(src, valid, m * R, d.nchunk, sums);
#pragma unroll
        for (int e = 0; e < E; ++e) {
            const int idx = base + e * kThreads;
            if (!valid[e]) continue;
            const int64_t i = i0 + idx / R;
            const int k = idx % R;
            if (p.dist) {
                // this rank's share of the all-reduce: the row's sum over its workers
                p.dist_out[d.prow_off + i * R + k] = sums[e];
                continue;
            }
            const double v = sums[e] * inv_w;
            pb_s[idx] = v;
            pbar[i * R + k] = v;
        }
    }
    if (tid == 0) cnt[cl.a_rb + tc.rb] = 0u;
    if (p.dist) return;
    __syncthreads();

    double* gram = p.ws.gram + d.gram_off;
    for (int pidx = tid; pidx < NG; pidx += kThreads) {
        int a = 0, rem = pidx;
        while (rem >= R - a) {
            rem -= R - a;
            ++a;
        }
        const int b = a + rem;
        double s = 0.0;
        for (int ii = 0; ii < rows; ++ii) s += pb_s[ii * R + a] * pb_s[ii * R + b];
        gram[static_cast<int64_t>(tc.rb) * NG + pidx] = s;
    }

    // 2) the last row block of a super-block: sum its Gram partials
    const int sup = tc.rb / kSuper;
    const int rb0 = sup * kSuper;
    const int nin = min(kSuper, d.nrb - rb0);
    __syncthreads();
    if (tid == 0) {
        __threadfence();
        const unsigned prev = atomicAdd(&cnt[cl.a_sup + sup], 1u);
        if (prev >= static_cast<unsigned>(nin)) atomicOr(p.ws.status, kStatusCounter);
        s_flag = (prev == static_cast<unsigned>(nin - 1));
    }
    __syncthreads();
    if (!s_flag) return;
    __threadfence();
    double* gsup = p.ws.gsup + d.gsup_off;
    for (int pidx = tid; pidx < NG; pidx += kThreads) {
        double s = sum_in_order(gram + static_cast<int64_t>(rb0) * NG + pidx, NG, nin);
        gsup[static_cast<int64_t>(sup) * NG + pidx] = s;
    }
    if (tid == 0) cnt[cl.a_sup + sup] = 0u;

    // 3) the last super-block of the layer: Gram sum and factorisation
    __syncthreads();
    if (tid == 0) {
        __threadfence();
        const unsigned prev = atomicAdd(&cnt[cl.a_layer], 1u);
        if (prev >= static_cast<unsigned>(d.nsup)) atomicOr(p.ws.status, kStatusCounter);
        s_flag = (prev == static_cast<unsigned>(d.nsup - 1));
    }
    __syncthreads();
    if (!s_flag) return;
    __threadfence();

    double* Gs = reinterpret_cast<double*>(fac);
    double* Rs = Gs + R * R;
    double* Ts = Rs + R * R;
    int* drop = reinterpret_cast<int*>(Ts + R * R);
    for (int pidx = tid; pidx < NG; pidx += kThreads) {
        int a = 0, rem = pidx;
        while (rem >= R - a) {
            rem -= R - a;
            ++a;
        }
        const int b = a + rem;
        double s = sum_in_order(gsup + pidx, NG, d.nsup);
        Gs[a * R + b] = s;
        Gs[b * R + a] = s;
    }
    __syncthreads();
    if (tid < 32) {
        factor_gram_warp<R>(Gs, Rs, Ts, drop, p.r, p.drop_tol, tid);
        double* T = p.ws.T + d.t_off;
        for (int idx = tid; idx < R * R; idx += 32) T[idx] = Ts[idx];
        if (p.track_conv && tid == 0 && p.iter >= 3) {
            // Subspace iteration on A = M_bar M_bar^T: from the second
            // iteration on, P_bar = A P_hat_prev, so the factor's diagonal
            // estimates the eigenvalues lambda_j = sigma_j^2 of A in
            // decreasing order.  The top r_conv directions of an r-column
            // block converge as (lambda_{r+1} / lambda_{r_conv})^iterations
            // (Halko, Martinsson and Tropp, SIAM Review 2011, section 4.5);
            // with the block's last estimate lambda_r standing in for
            // lambda_{r+1} >= ..., the layer stops after this iteration once
            // that factor is at most conv_eps.  A zero lambda_{r_conv} (rank
            // below r_conv: the range is captured exactly) stops it too.
            const double lam_keep = Rs[(p.r_conv - 1) * R + (p.r_conv - 1)];
            const double lam_last = Rs[(p.r - 1) * R + (p.r - 1)];
            const bool done = !(lam_keep > 0.0) || pow(lam_last / lam_keep, p.iter - 1) <= p.conv_eps;
            if (done) p.ws.conv_iter[tc.l] = p.iter;
        }
    }
    if (tid == 0) cnt[cl.a_layer] = 0u;
}

// READM: a later power iteration of the same step; M is already in the
// error buffers, so only M is read (no gradient, no store).
template <int R, typename GT, bool LAZY, bool SF, bool READM>
__global__ void __launch_bounds__(kThreads, (R <= 8 ? 3 : 2)) k_pass_a(Params p) {
    extern __shared__ __align__(16) unsigned char smem[];
    const int t = p.tile_base + tile_index<false>();
    const int l = p.t.tile_layer[t];
    if (p.track_conv && p.iter > p.ws.conv_iter[l]) return;   // converged refresh layer
    const LayerDesc d = p.t.layers[l];
    const TileCoord tc = decode_tile(d, t, l);
    const int W = p.workers;
    const int L = p.num_layers;

    const GT** gp = reinterpret_cast<const GT**>(smem);
    float** ep = reinterpret_cast<float**>(smem + static_cast<size_t>(W) * sizeof(void*));
    double* rows_d = reinterpret_cast<double*>(smem + ((SmemA<R>::ptr_bytes(W) + 15) & ~size_t(15)));
    float* rows_s = reinterpret_cast<float*>(rows_d);
    unsigned char* fac = reinterpret_cast<unsigned char*>(rows_d) + ((SmemA<R>::rows_bytes(d.tm) + 15) & ~size_t(15));
    float* wide = reinterpret_cast<float*>(fac + ((SmemA<R>::fac_bytes() + 15) & ~size_t(15)));

    for (int w = threadIdx.x; w < W; w += kThreads) {
        gp[w] = static_cast<const GT*>(p.t.grads[w * L + l]);
        ep[w] = p.t.errors[w * L + l];
    }
    if constexpr (LAZY) {
        const int64_t i0 = static_cast<int64_t>(tc.rb) * d.tm;
        const int rows = static_cast<int>(min(static_cast<int64_t>(d.tm), d.m - i0));
        const float* ph = p.ws.phat + d.prow_off + i0 * R;
        for (int idx = threadIdx.x; idx < rows * R; idx += kThreads) rows_s[idx] = p.use_prev ? ph[idx] : 0.f;
    }
    __syncthreads();

    if constexpr (UseMma<R>::value) {
        unsigned char* wb = reinterpret_cast<unsigned char*>(wide);
        if (d.vec == 4) {
            pass_a_mma<R, 4, GT, LAZY, SF, READM>(p, d, tc, gp, ep, rows_s, wb);
        } else if (d.vec == 2) {
            pass_a_mma<R, 2, GT, LAZY, SF, READM>(p, d, tc, gp, ep, rows_s, wb);
        } else {
            pass_a_mma<R, 1, GT, LAZY, SF, READM>(p, d, tc, gp, ep, rows_s, wb);
        }
    } else {
        // VEC x R values of Q live in registers: VEC = 4 up to R = 4, 2 up to 16
        if (d.vec == 4) {
            if constexpr (R <= 4) pass_a_rows<R, 4, GT, LAZY, SF, READM>(p, d, tc, gp, ep, rows_s);
        } else if (d.vec == 2) {
            if constexpr (R <= 16) pass_a_rows<R, 2, GT, LAZY, SF, READM>(p, d, tc, gp, ep, rows_s);
        } else {
            pass_a_rows<R, 1, GT, LAZY, SF, READM>(p, d, tc, gp, ep, rows_s);
        }
    }
    pass_a_epilogue<R>(p, d, tc, rows_d, fac);
}

// ---------------------------------------------------------------------------
// pass B

template <int R>
struct SmemB {
    static __host__ __device__ size_t ptr_bytes(int W) { return static_cast<size_t>(W) * sizeof(void*); }
    static __host__ __device__ size_t rows_bytes(int tm) { return static_cast<size_t>(tm) * R * sizeof(float); }
    static __host__ __device__ size_t red_bytes(int vec) {
        if (UseMma<R>::value && vec == 4) {
            // staged kernel: the M stages, reused at the end for the warps'
            // partials (8 warps x 64 columns x (R + 1) floats)
            const size_t red = static_cast<size_t>(kWarps) * 64 * (R + 1) * sizeof(float);
            const size_t staged = kStgBytes > red ? kStgBytes : red;
            return staged > TcSmem<R>::total ? staged : TcSmem<R>::total;
        }
        if (UseMma<R>::value) {
            // tensor-core kernel: warp partials (8 x 32 columns x 33) + the
            // warps' A fragments
            return static_cast<size_t>(kWarps) * kWideCols * kRedStride * sizeof(float) + kPaBytes;
        }
        return static_cast<size_t>(kWarps) * R * vec * 32 * sizeof(float);
    }
    static __host__ __device__ size_t total(int W, int tm, int vec) {
        return ((ptr_bytes(W) + 15) & ~size_t(15)) + ((rows_bytes(tm) + 15) & ~size_t(15)) + red_bytes(vec);
    }
};

// The tile's P_hat rows [i0, i0+rows) from the workspace (formed once per
// layer by k_phat) into shared memory; a thread's loads are all in flight
// together.
template <int R>
__device__ __forceinline__ void load_phat_rows(const Params& p, const LayerDesc& d, const TileCoord& tc,
                                               float* ph_s) {
    constexpr int kE = kRowsFloatsMax / kThreads;   // elements per thread at most
    const int64_t i0 = static_cast<int64_t>(tc.rb) * d.tm;
    const int rows = static_cast<int>(min(static_cast<int64_t>(d.tm), d.m - i0));
    const int total = rows * R;
    const float* src = p.ws.phat + d.prow_off + i0 * R;
    float v[kE];
#pragma unroll
    for (int e = 0; e < kE; ++e) {
        const int idx = threadIdx.x + e * kThreads;
        v[e] = idx < total ? __ldg(src + idx) : 0.f;
    }
#pragma unroll
    for (int e = 0; e < kE; ++e) {
        const int idx = threadIdx.x + e * kThreads;
        if (idx < total) ph_s[idx] = v[e];
    }
    __syncthreads();
}

template <int R, int VEC, bool SF>
__device__ __forceinline__ void pass_b_rows(const Params& p, const LayerDesc& d, const TileCoord& tc,
                                            float* const* ep, const float* ph_s, float* red_s) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int W = p.workers;
    const int64_t n = d.n, m = d.m;
    const int64_t i0 = static_cast<int64_t>(tc.rb) * d.tm;
    const int64_t i1 = min(i0 + d.tm, m);
    const int s0 = tc.c * d.slots;
    const int ns = min(d.slots, d.nvec - s0);
    const bool active = lane < ns;
    const int64_t j = static_cast<int64_t>(s0 + (active ? lane : 0)) * VEC;
    // pass B only reads: 128 bytes of loads in flight per lane (8, 16 or 32
    // workers for 16-, 8- and 4-byte lanes)
    constexpr int U = 32 / VEC;

    float qacc[VEC][R];
#pragma unroll
    for (int v = 0; v < VEC; ++v)
#pragma unroll
        for (int k = 0; k < R; ++k) qacc[v][k] = 0.f;

    if (active && W <= 4) {
        // few workers: two rows' loads in flight together, then the
        // products in the same order as the loop below (row, then worker)
        for (int64_t i = i0 + warp; i < i1; i += 2 * kWarps) {
            const bool two = i + kWarps < i1;
            float e[2][4][VEC];
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    if (u < W && (h == 0 || two)) ld_f32<VEC>(ep[u] + (i + h * kWarps) * n + j, e[h][u]);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                if (h == 1 && !two) break;
                float ph[R];
#pragma unroll
                for (int k = 0; k < R; ++k) ph[k] = ph_s[(i + h * kWarps - i0) * R + k];
                float msum[VEC];
#pragma unroll
                for (int v = 0; v < VEC; ++v) msum[v] = 0.f;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    if (u < W) {
                        if constexpr (SF) {
#pragma unroll
                            for (int v = 0; v < VEC; ++v) msum[v] += e[h][u][v];
                        } else {
#pragma unroll
                            for (int v = 0; v < VEC; ++v) axpy<R>(qacc[v], e[h][u][v], ph);
                        }
                    }
                }
                if constexpr (SF) {
#pragma unroll
                    for (int v = 0; v < VEC; ++v) axpy<R>(qacc[v], msum[v], ph);
                }
            }
        }
    } else if (active) {
        for (int64_t i = i0 + warp; i < i1; i += kWarps) {
            float ph[R];
#pragma unroll
            for (int k = 0; k < R; ++k) ph[k] = ph_s[(i - i0) * R + k];
            const int64_t base = i * n + j;
            float msum[VEC];
#pragma unroll
            for (int v = 0; v < VEC; ++v) msum[v] = 0.f;
            // G workers' loads in flight, then their products
            auto group = [&](auto GC, int w0) {
                constexpr int G = decltype(GC)::value;
                float e[G][VEC];
#pragma unroll
                for (int u = 0; u < G; ++u) ld_f32<VEC>(ep[w0 + u] + base, e[u]);
#pragma unroll
                for (int u = 0; u < G; ++u) {
                    if constexpr (SF) {
#pragma unroll
                        for (int v = 0; v < VEC; ++v) msum[v] += e[u][v];
                    } else {
#pragma unroll
                        for (int v = 0; v < VEC; ++v) axpy<R>(qacc[v], e[u][v], ph);
                    }
                }
            };
            int w = 0;
            for (; w + U <= W; w += U) group(std::integral_constant<int, U>{}, w);
            if constexpr (U > 16) {
                if (w + 16 <= W) {
                    group(std::integral_constant<int, 16>{}, w);
                    w += 16;
                }
            }
            if constexpr (U > 8) {
                if (w + 8 <= W) {
                    group(std::integral_constant<int, 8>{}, w);
                    w += 8;
                }
            }
            if (w + 4 <= W) {
                group(std::integral_constant<int, 4>{}, w);
                w += 4;
            }
            if (w + 2 <= W) {
                group(std::integral_constant<int, 2>{}, w);
                w += 2;
            }
            if (w < W) group(std::integral_constant<int, 1>{}, w);
            if constexpr (SF) {
#pragma unroll
                for (int v = 0; v < VEC; ++v)
                    axpy<R>(qacc[v], msum[v], ph);
            }
        }
    }
    // this warp's partial, laid out [warp][k][v][lane] (conflict-free)
#pragma unroll
    for (int k = 0; k < R; ++k)
#pragma unroll
        for (int v = 0; v < VEC; ++v) red_s[((warp * R + k) * VEC + v) * 32 + lane] = qacc[v][k];
    __syncthreads();
    // sum over warps in order; write the row block's partial Q rows
    double* qpart = p.ws.qpart + d.qpart_off;
    const int cols = ns * VEC;
    for (int idx = threadIdx.x; idx < cols * R; idx += kThreads) {
        const int cc = idx / R;        // local column
        const int k = idx % R;
        const int ln = cc / VEC, v = cc % VEC;
        double s = 0.0;
#pragma unroll
        for (int wp = 0; wp < kWarps; ++wp) s += static_cast<double>(red_s[((wp * R + k) * VEC + v) * 32 + ln]);
        qpart[(static_cast<int64_t>(tc.rb) * n + static_cast<int64_t>(s0) * VEC + cc) * R + k] = s;
    }
}

// Tensor-core variant of the second pass (R = 32).  Warps split as in the
// first pass: a row group of 16 rows per warp, the row group's warps
// ("parts") dealing the workers.  The Q partial of a sub-chunk is
// D (32 ranks x 32 columns) = P_hat^T (ranks x rows) * M (rows x columns):
// the A fragments (P_hat^T of the warp's rows, split into tf32 hi and lo)
// are formed once per tile in shared memory; the B fragments are M itself,
// loaded straight from global memory.  Column order: lane (g, t) loads
// columns 4g .. 4g + 3 of the rows it needs, and n-tile j takes column
// 4g + j as its column g.  D accumulates in float32 over the warp's rows
// and workers (one sub-chunk at a time); the 8 warps' D are then summed in
// float64 in warp order, as in the CUDA-core passes.

// Row ii (tile row) of M for the 32 columns of a sub-chunk, in the lane's
// four columns 4g .. 4g + 3 (zero outside the layer).
template <int VEC>
__device__ __forceinline__ void load_cols4(const float* rp, bool ok, int c, int cols, float (&x)[4]) {
    x[0] = x[1] = x[2] = x[3] = 0.f;
    if (!ok) return;
    if constexpr (VEC == 4) {
        if (c < cols) ld_f32<4>(rp + c, x);
    } else if constexpr (VEC == 2) {
#pragma unroll
        for (int h = 0; h < 2; ++h)
            if (c + 2 * h < cols) {
                float y[2];
                ld_f32<2>(rp + c + 2 * h, y);
                x[2 * h] = y[0];
                x[2 * h + 1] = y[1];
            }
    } else {
#pragma unroll
        for (int h = 0; h < 4; ++h)
            if (c + h < cols) x[h] = rp[c + h];
    }
}

template <int R, int VEC, bool SF>
__device__ __forceinline__ void pass_b_mma(const Params& p, const LayerDesc& d, const TileCoord& tc,
                                           float* const* ep, const float* ph_s, float* red_s) {
    static_assert(R == 16 || R == 32, "tensor-core pass B: rank 16 or 32");
    constexpr int MT = R / 16;                  // m-tiles of 16 ranks
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, t4 = lane & 3;
    const int W = p.workers;
    const int64_t n = d.n;
    const int64_t i0 = static_cast<int64_t>(tc.rb) * d.tm;
    const int rows = static_cast<int>(min(static_cast<int64_t>(d.tm), d.m - i0));
    const int64_t jc = static_cast<int64_t>(tc.c) * d.slots * d.vec;
    const int width = static_cast<int>(min(static_cast<int64_t>(d.slots) * d.vec, n - jc));
    const int nsc = (width + kWideCols - 1) / kWideCols;
    const int nrg = d.tm / kMmaRows;
    const int parts = kWarps / nrg;
    const int rg = warp % nrg, part = warp / nrg;
    const int r0 = rg * kMmaRows;
    double* qpart = p.ws.qpart + d.qpart_off;
    float4* pa = reinterpret_cast<float4*>(red_s + kWarps * kWideCols * kRedStride);   // [warp][ks][mt][lane][hi, lo]

    // A fragments of this warp: A[rank][row] = P_hat[r0 + row][rank], rows
    // outside the layer zero; slot t <- row 8 ks + t, slot t + 4 <- row 8 ks + t + 4
#pragma unroll
    for (int ks = 0; ks < 2; ++ks)
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
            float av[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int row = r0 + 8 * ks + t4 + 4 * (q >> 1);
                const int rank = 16 * mt + g + 8 * (q & 1);
                av[q] = row < rows ? ph_s[row * R + rank] : 0.f;
            }
            uint32_t hi[4], lo[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) tf32_split(av[q], hi[q], lo[q]);
            float4* dst = pa + (((warp * 2 + ks) * MT + mt) * 32 + lane) * 2;
            dst[0] = make_float4(__uint_as_float(hi[0]), __uint_as_float(hi[1]), __uint_as_float(hi[2]),
                                 __uint_as_float(hi[3]));
            dst[1] = make_float4(__uint_as_float(lo[0]), __uint_as_float(lo[1]), __uint_as_float(lo[2]),
                                 __uint_as_float(lo[3]));
        }
    __syncwarp();

    // this part's workers: part, part + parts, ...
    const int nw = W > part ? (W - part + parts - 1) / parts : 0;
    const int64_t row0 = (i0 + r0) * n + jc;
    // the lane's rows: 8 ks + t4 and 8 ks + t4 + 4 (tile rows r0 + ...)
    auto load = [&](int sc, int w, float (&mv)[2][2][4]) {
        const int cols = width - sc * kWideCols;
#pragma unroll
        for (int ks = 0; ks < 2; ++ks)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int row = 8 * ks + t4 + 4 * hh;
                load_cols4<VEC>(ep[w] + row0 + static_cast<int64_t>(row) * n + sc * kWideCols, r0 + row < rows,
                                4 * g, cols, mv[ks][hh]);
            }
    };

    float cur[2][2][4], nxt[2][2][4];
    float msum[SF ? 2 : 1][SF ? 2 : 1][SF ? 4 : 1];
    if (nw > 0) load(0, part, nxt);
    for (int sc = 0; sc < nsc; ++sc) {
        float dacc[MT][4][4];   // [m-tile][n-tile][fragment]
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int q = 0; q < 4; ++q) dacc[mt][nt][q] = 0.f;
        if constexpr (SF) {
#pragma unroll
            for (int ks = 0; ks < 2; ++ks)
#pragma unroll
                for (int hh = 0; hh < 2; ++hh)
#pragma unroll
                    for (int j = 0; j < 4; ++j) msum[ks][hh][j] = 0.f;
        }
        for (int wi = 0; wi < nw; ++wi) {
#pragma unroll
            for (int ks = 0; ks < 2; ++ks)
#pragma unroll
                for (int hh = 0; hh < 2; ++hh)
#pragma unroll
                    for (int j = 0; j < 4; ++j) cur[ks][hh][j] = nxt[ks][hh][j];
            // next (sub-chunk, worker) in flight while this block is multiplied
            if (wi + 1 < nw) load(sc, part + (wi + 1) * parts, nxt);
            else if (sc + 1 < nsc) load(sc + 1, part, nxt);
            bool go = true;
            if constexpr (SF) {
#pragma unroll
                for (int ks = 0; ks < 2; ++ks)
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh)
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            msum[ks][hh][j] += cur[ks][hh][j];
                            cur[ks][hh][j] = msum[ks][hh][j];
                        }
                go = wi == nw - 1;
            }
            if (go) {
#pragma unroll
                for (int ks = 0; ks < 2; ++ks) {
                    // B fragments of the four n-tiles: b0 = row t4, b1 = row t4 + 4
                    uint32_t bh[4][2], bl[4][2];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        tf32_split(cur[ks][0][j], bh[j][0], bl[j][0]);
                        tf32_split(cur[ks][1][j], bh[j][1], bl[j][1]);
                    }
#pragma unroll
                    for (int mt = 0; mt < MT; ++mt) {
                        const float4* src = pa + (((warp * 2 + ks) * MT + mt) * 32 + lane) * 2;
                        const float4 h4 = src[0], l4 = src[1];
                        const uint32_t ahi[4] = {__float_as_uint(h4.x), __float_as_uint(h4.y), __float_as_uint(h4.z),
                                                 __float_as_uint(h4.w)};
                        const uint32_t alo[4] = {__float_as_uint(l4.x), __float_as_uint(l4.y), __float_as_uint(l4.z),
                                                 __float_as_uint(l4.w)};
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            mma_tf32(dacc[mt][j], alo, bh[j][0], bh[j][1]);
                            mma_tf32(dacc[mt][j], ahi, bl[j][0], bl[j][1]);
                            mma_tf32(dacc[mt][j], ahi, bh[j][0], bh[j][1]);
                        }
                    }
                }
            }
        }
        // sub-chunk done: every warp's D to shared memory, then summed over
        // the warps in warp order (float64) per (column, rank)
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int rank = 16 * mt + g + 8 * (q >> 1);
                    const int col = 4 * (2 * t4 + (q & 1)) + j;
                    red_s[(warp * kWideCols + col) * kRedStride + rank] = dacc[mt][j][q];
                }
        __syncthreads();
        const int ncols = min(kWideCols, width - sc * kWideCols);
        for (int idx = tid; idx < ncols * R; idx += kThreads) {
            const int c = idx / R, kk = idx % R;
            double s2 = 0.0;
#pragma unroll
            for (int wp = 0; wp < kWarps; ++wp) s2 += static_cast<double>(red_s[(wp * kWideCols + c) * kRedStride + kk]);
            qpart[(static_cast<int64_t>(tc.rb) * n + jc + sc * kWideCols + c) * R + kk] = s2;
        }
        __syncthreads();
    }
}

// Staged second pass for R = 16, 32 with 16-byte rows (n % 4 == 0), on the
// CUDA cores.  The tile (tm <= 64 rows x a chunk of <= 128 columns) is
// processed one worker at a time: the worker's block is copied into a
// shared-memory stage by cp.async while the previous worker's block is
// multiplied, so that 32 KB blocks are in flight without holding registers.
// Warp w takes the chunk columns 64 (w & 1) .. 64 (w & 1) + 63 and the tile
// rows (w >> 1) + 4 i.  Lane l takes 4 columns, 4 (l % 16) .. + 3 of that
// half, and half of the ranks, R / 2 (l / 16) .. + R / 2 - 1: per row, one
// 16-byte load of M and R / 8 broadcast 16-byte loads of the P_hat row feed
// 2 R fused multiply-adds (packed, two ranks per instruction, accumulators
// kept as pairs), summed in float32 over the warp's rows and the workers.
// (Measured on the B200, the tf32 mma.sync path needs three split products
// per term and its tensor pipe saturated at the CUDA cores' multiply-add
// rate.)  At the end the four row-quarter warps of each column half are
// added in float64, in order.
template <int R, bool SF>
__device__ __forceinline__ void pass_b_staged(const Params& p, const LayerDesc& d, const TileCoord& tc,
                                              float* const* ep, const float* ph_s, float* red_s) {
    static_assert(R == 16 || R == 32, "staged pass B: rank 16 or 32");
    constexpr int RH = R / 2;                   // ranks per lane
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int W = p.workers;
    const int64_t n = d.n;
    const int64_t i0 = static_cast<int64_t>(tc.rb) * d.tm;
    const int rows = static_cast<int>(min(static_cast<int64_t>(d.tm), d.m - i0));
    const int64_t jc = static_cast<int64_t>(tc.c) * d.slots * 4;
    const int width = static_cast<int>(min(static_cast<int64_t>(d.slots) * 4, n - jc));
    float* stg = red_s;                         // [stage][row][kStgStride]
    const int half = warp & 1, rq = warp >> 1;
    const int lc = 64 * half + 4 * (lane & 15); // the lane's first column in the chunk
    const int k0 = RH * (lane >> 4);            // the lane's first rank
    const bool active = lc < width;

    // one worker's block into stage s: (tm rows) x (32 x 16 bytes)
    auto issue = [&](int w, int stage) {
        float* dst = stg + static_cast<size_t>(stage) * kStgRows * kStgStride;
        const float* src = ep[w] + i0 * n + jc;
        for (int idx = tid; idx < d.tm * (kStgCols / 4); idx += kThreads) {
            const int row = idx >> 5, c4 = (idx & 31) * 4;
            const bool ok = row < rows && c4 < width;
            cp_async16(dst + row * kStgStride + c4, ok ? src + static_cast<int64_t>(row) * n + c4 : src, ok);
        }
    };

    float2 acc[4][RH / 2];                      // [column][rank pair]
#pragma unroll
    for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int k = 0; k < RH / 2; ++k) acc[c][k] = make_float2(0.f, 0.f);
    float4 msum[SF ? kStgRows / 4 : 1];
    if constexpr (SF) {
#pragma unroll
        for (int i = 0; i < kStgRows / 4; ++i) msum[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    auto rank_update = [&](const float4 x, int row) {
        const float4* ph4 = reinterpret_cast<const float4*>(ph_s + row * R + k0);
        const float2 xs[4] = {make_float2(x.x, x.x), make_float2(x.y, x.y), make_float2(x.z, x.z),
                              make_float2(x.w, x.w)};
#pragma unroll
        for (int k4 = 0; k4 < RH / 4; ++k4) {
            const float4 pv = ph4[k4];
            const float2 p01 = make_float2(pv.x, pv.y), p23 = make_float2(pv.z, pv.w);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                acc[c][2 * k4] = __ffma2_rn(xs[c], p01, acc[c][2 * k4]);
                acc[c][2 * k4 + 1] = __ffma2_rn(xs[c], p23, acc[c][2 * k4 + 1]);
            }
        }
    };

    // pipeline over the workers: kStages - 1 blocks ahead
#pragma unroll
    for (int s0 = 0; s0 < kStages - 1; ++s0) {
        if (s0 < W) issue(s0, s0);
        cp_async_commit();
    }
    for (int w = 0; w < W; ++w) {
        const int ahead = w + kStages - 1;
        if (ahead < W) issue(ahead, ahead % kStages);
        cp_async_commit();                       // (an empty group keeps the count uniform)
        cp_async_wait<kStages - 1>();            // worker w's block has landed
        __syncthreads();
        const float* blk = stg + static_cast<size_t>(w % kStages) * kStgRows * kStgStride;
        if (active) {
#pragma unroll 2
            for (int i = 0; i < kStgRows / 4; ++i) {
                const int row = rq + 4 * i;
                if (row < rows) {
                    const float4 x = *reinterpret_cast<const float4*>(blk + row * kStgStride + lc);
                    if constexpr (SF) {
                        msum[i].x += x.x;
                        msum[i].y += x.y;
                        msum[i].z += x.z;
                        msum[i].w += x.w;
                        if (w == W - 1) rank_update(msum[i], row);
                    } else {
                        rank_update(x, row);
                    }
                }
            }
        }
        __syncthreads();   // stage w % kStages may be refilled next
    }
    cp_async_wait<0>();

    // the four row quarters of each column half, in float64 and in order;
    // the stages are free now: red[warp][col (64)][R + 1] floats
    constexpr int RS = R + 1;
    float* red = stg;
    const int cl = 4 * (lane & 15);
#pragma unroll
    for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int k = 0; k < RH / 2; ++k) {
            red[(warp * 64 + cl + c) * RS + k0 + 2 * k] = acc[c][k].x;
            red[(warp * 64 + cl + c) * RS + k0 + 2 * k + 1] = acc[c][k].y;
        }
    __syncthreads();
    double* qpart = p.ws.qpart + d.qpart_off;
    for (int idx = tid; idx < width * R; idx += kThreads) {
        const int col = idx / R, k = idx - (idx / R) * R;
        const int h = col >> 6, c = col & 63;
        double s2 = 0.0;
#pragma unroll
        for (int q = 0; q < 4; ++q) s2 += static_cast<double>(red[((2 * q + h) * 64 + c) * RS + k]);
        qpart[(static_cast<int64_t>(tc.rb) * n + jc + col) * R + k] = s2;
    }
}

// Second pass on the 5th-generation tensor cores (R = 16, 32; 16-byte rows).
// For every worker, D (128 chunk columns x ranks, float32, in tensor memory)
// = M^T P_hat over the tile's rows.  A = the worker's block of M, K-major in
// tensor memory: each thread owns one TMEM lane (a chunk column) and half
// of the tile's rows; it loads its 32 rows one worker ahead into registers
// (a warp's loads take 128 contiguous bytes of a row), splits them into hi
// (the top 19 bits) and lo = x - hi, and writes both with tcgen05.st.
// B = [P_hat hi | P_hat lo] (round-to-nearest split), K-major in shared
// memory, once per tile.  Per k-step of 8 rows two MMAs give fp32 accuracy
// from tf32 products (split-precision products, Markidis et al. 2018):
// A_hi [B_hi | B_lo] (N = 2R) and A_lo B_hi (N = R, accumulated into the
// first half), so D = [hi*hi + lo*hi | hi*lo], in kTcChains independent
// accumulators (k-step ks into ks % kTcChains).  Warp 0 runs the issue loop,
// one elected lane issues them and commits to an mbarrier, and one thread
// waits on it before the next worker's block is written.  D accumulates
// over groups of kTcGroup workers; after each group all eight warps read it
// back (tcgen05.ld: four lane quarters x two rank halves; chains and halves
// summed in float32) into float64 sums (each thread's own slots in shared
// memory), so float32 runs stay within kTcGroup workers' rows of one tile.
// Every wait is bounded (about a
// second), after which the status word is set and the tile winds down; the
// tensor memory is released on every path.

__device__ __forceinline__ uint32_t tc_kmajor(int mn, int k, uint32_t sbo) {   // bytes; K extent 64
    return static_cast<uint32_t>((mn >> 3) * sbo + (k >> 2) * 128 + (mn & 7) * 16 + (k & 3) * 4);
}

// 32 TMEM lanes x N consecutive columns (N = 8 or 16) into this warp; the
// values are valid after tmem_wait_ld()
template <int N>
__device__ __forceinline__ void tmem_ld(uint32_t taddr, uint32_t (&u)[N]) {
    if constexpr (N == 16) {
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
            "%14, %15}, [%16];"
            : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]), "=r"(u[7]),
              "=r"(u[8]), "=r"(u[9]), "=r"(u[10]), "=r"(u[11]), "=r"(u[12]), "=r"(u[13]), "=r"(u[14]), "=r"(u[15])
            : "r"(taddr));
    } else {
        static_assert(N == 8, "tmem_ld: 8 or 16 columns");
        asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                     : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]),
                       "=r"(u[7])
                     : "r"(taddr));
    }
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

template <int R>
__device__ __forceinline__ void pass_b_tc(const Params& p, const LayerDesc& d, const TileCoord& tc,
                                          float* const* ep, const float* ph_s, unsigned char* buf) {
    static_assert(R == 16 || R == 32, "tensor-core pass B: rank 16 or 32");
    constexpr int RH = R / 2;   // ranks per reading warp
    constexpr int KH = 32;      // rows of K per thread (half of the 64-row tile)
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int W = p.workers;
    const int64_t n = d.n;
    const int64_t i0 = static_cast<int64_t>(tc.rb) * d.tm;
    const int rows = static_cast<int>(min(static_cast<int64_t>(d.tm), d.m - i0));
    const int64_t jc = static_cast<int64_t>(tc.c) * d.slots * 4;
    const int width = static_cast<int>(min(static_cast<int64_t>(d.slots) * 4, n - jc));
    const int nks = d.tm / 8;
    unsigned char* b_s = buf;
    double* dsum = reinterpret_cast<double*>(b_s + TcSmem<R>::b_bytes);   // [RH][kThreads]
    uint64_t* bar = reinterpret_cast<uint64_t*>(b_s + TcSmem<R>::b_bytes + TcSmem<R>::sum_bytes);
    uint32_t* tslot = reinterpret_cast<uint32_t*>(bar + 1);
    int* flag = reinterpret_cast<int*>(tslot + 1);
    const uint32_t bar_a = static_cast<uint32_t>(__cvta_generic_to_shared(bar));
    constexpr uint32_t kIdescHL = umma_idesc_tf32(128, 2 * R);
    constexpr uint32_t kIdescL = umma_idesc_tf32(128, R);

    // this thread: TMEM lane (chunk column) 32 (warp & 3) + lane, rows
    // KH (warp >> 2) .. + KH - 1 of the tile
    const int col = (warp & 3) * 32 + lane;
    const int r0 = KH * (warp >> 2);
    const bool has_rows = r0 < d.tm;   // uniform over the warp
    const bool col_ok = col < width;
    const int nr = col_ok ? max(0, min(KH, rows - r0)) : 0;   // rows this thread loads
    auto load = [&](int w, float (&v)[KH]) {
        const float* src = ep[w] + (i0 + r0) * n + jc + col;
#pragma unroll
        for (int r = 0; r < KH; ++r) {
            v[r] = r < nr ? __ldcg(src) : 0.f;
            src += n;
        }
    };

    // set-up: barrier, tensor memory, B
    if (tid == 0) {
        mbar_init(bar_a, 1);
        *flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         static_cast<uint32_t>(__cvta_generic_to_shared(tslot))),
                     "r"(TcSmem<R>::tmem_cols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    for (int idx = tid; idx < d.tm * R; idx += kThreads) {
        const int row = idx / R, k = idx - (idx / R) * R;
        uint32_t hi = 0, lo = 0;
        if (row < rows) tf32_split(ph_s[row * R + k], hi, lo);
        *reinterpret_cast<uint32_t*>(b_s + tc_kmajor(k, row, kTcSboB)) = hi;
        *reinterpret_cast<uint32_t*>(b_s + tc_kmajor(R + k, row, kTcSboB)) = lo;
    }
    float x[KH], xn[KH];
    if (W > 0 && has_rows) load(0, x);
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);   // this warp's TMEM lanes

    // hi and lo of this thread's rows into its TMEM lane (v is left holding lo)
    auto store_a = [&](float (&v)[KH]) {
#pragma unroll
        for (int j = 0; j < KH; j += 8) {
            uint32_t u[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                u[k] = __float_as_uint(v[j + k]) & 0xffffe000u;
                v[j + k] -= __uint_as_float(u[k]);
            }
            tmem_st8(t_lane + kTcAHi + static_cast<uint32_t>(r0 + j), u);
        }
#pragma unroll
        for (int j = 0; j < KH; j += 8) {
            uint32_t u[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) u[k] = __float_as_uint(v[j + k]);
            tmem_st8(t_lane + kTcALo + static_cast<uint32_t>(r0 + j), u);
        }
        tmem_wait_st();
    };

#pragma unroll
    for (int k = 0; k < RH; ++k) dsum[k * kThreads + tid] = 0.0;   // this thread's own slots
    const int kh = (warp >> 2) * RH;   // this warp's ranks
    // the chains' two halves summed in float32 (chains beyond the tile's
    // k-steps hold nothing), then added to the float64 sums; 8 ranks at a time
    auto read_back = [&]() {
#pragma unroll
        for (int k0 = 0; k0 < RH; k0 += 8) {
            uint32_t u[8];
            float f[8];
            tmem_ld<8>(t_lane + kTcD + static_cast<uint32_t>(kh + k0), u);   // chain 0, hi*hi + lo*hi
            tmem_wait_ld();
#pragma unroll
            for (int k = 0; k < 8; ++k) f[k] = __uint_as_float(u[k]);
#pragma unroll
            for (int c = 0; c < kTcChains; ++c)
#pragma unroll
                for (int h = (c == 0 ? 1 : 0); h < 2; ++h) {
                    if (c < nks) {   // uniform over the block
                        tmem_ld<8>(t_lane + kTcD + static_cast<uint32_t>(c * 2 * R + h * R + kh + k0), u);
                        tmem_wait_ld();
#pragma unroll
                        for (int k = 0; k < 8; ++k) f[k] += __uint_as_float(u[k]);
                    }
                }
#pragma unroll
            for (int k = 0; k < 8; ++k) dsum[(k0 + k) * kThreads + tid] += static_cast<double>(f[k]);
        }
    };
    // one thread waits for worker w's products; the others at the barrier
    auto wait_products = [&](int w) -> bool {
        if (tid == 0 && !mbar_wait_bounded(bar_a, static_cast<uint32_t>(w & 1), p.ws.status)) *flag = 1;
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        return *flag == 0;
    };

    // worker w: its rows are in `cur`; the next worker's are loaded into
    // `nxt` (the two register sets alternate, so no copy waits on the loads)
    bool ok = true;
    auto worker = [&](int w, float (&cur)[KH], float (&nxt)[KH]) -> bool {
        if (w + 1 < W && has_rows) load(w + 1, nxt);
        if (w > 0) {
            // worker w - 1's products are done: A and D are free
            if (!wait_products(w - 1)) return false;
            if ((w - 1) % kTcGroup == kTcGroup - 1) read_back();
        }
        if (has_rows) store_a(cur);
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (warp == 0 && !p.stall_products) {
            // warp-uniform loop; one elected lane issues
            const bool leader = elect_one();
            const uint32_t acc0 = (w % kTcGroup) ? 1u : 0u;
            const uint32_t bb = static_cast<uint32_t>(__cvta_generic_to_shared(b_s));
            for (int ks = 0; ks < nks; ++ks) {
                const uint32_t dc = tmem + kTcD + static_cast<uint32_t>((ks % kTcChains) * 2 * R);
                if (leader) {
                    // 8 rows of K: 8 TMEM columns of A, two K core matrices (256 bytes) of B
                    const uint64_t db = umma_desc(bb + static_cast<uint32_t>(ks) * 256, 128, kTcSboB);
                    umma_tf32_ts(dc, tmem + kTcAHi + static_cast<uint32_t>(ks) * 8, db, kIdescHL,
                                 ks >= kTcChains ? 1u : acc0);
                    umma_tf32_ts(dc, tmem + kTcALo + static_cast<uint32_t>(ks) * 8, db, kIdescL, 1u);
                }
            }
            if (leader) umma_commit(bar_a);
            __syncwarp();
        }
        return true;
    };
    for (int w = 0; w < W && ok; w += 2) {
        ok = worker(w, x, xn);
        if (ok && w + 1 < W) ok = worker(w + 1, xn, x);
    }
    if (ok && W > 0) {
        ok = wait_products(W - 1);
        if (ok) read_back();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TcSmem<R>::tmem_cols)
                     : "memory");
    }
    if (!ok) return;   // the status word says why; this tile's partial is not written
    // this thread's chunk column (TMEM lane) and rank half of the row block's partial Q rows
    if (col_ok) {
        double* qp = p.ws.qpart + d.qpart_off + (static_cast<int64_t>(tc.rb) * n + jc + col) * R + kh;
#pragma unroll
        for (int k = 0; k < RH; ++k) qp[k] = dsum[k * kThreads + tid];
    }
}

template <int R>
__device__ void pass_b_epilogue(const Params& p, const LayerDesc& d, const TileCoord& tc) {
    __shared__ int s_flag;
    const int tid = threadIdx.x;
    const CounterLayout cl = counter_layout(d.nrb, d.nsup, d.nchunk);
    unsigned* cnt = p.ws.cnt + d.cnt_off;
    const int64_t n = d.n;
    const int s0 = tc.c * d.slots;
    const int ns = min(d.slots, d.nvec - s0);
    const int64_t col0 = static_cast<int64_t>(s0) * d.vec;
    const int cols = ns * d.vec;

    // 1) the last row block of a super-block (for this chunk): sum its partials
    const int sup = tc.rb / kSuper;
    const int rb0 = sup * kSuper;
    const int nin = min(kSuper, d.nrb - rb0);
    unsigned* c1 = &cnt[cl.b_sup + static_cast<int64_t>(tc.c) * d.nsup + sup];
    __syncthreads();
    if (tid == 0) {
        __threadfence();
        const unsigned prev = atomicAdd(c1, 1u);
        if (prev >= static_cast<unsigned>(nin)) atomicOr(p.ws.status, kStatusCounter);
        s_flag = (prev == static_cast<unsigned>(nin - 1));
    }
    __syncthreads();
    if (!s_flag) return;
    __threadfence();
    const double* qpart = p.ws.qpart + d.qpart_off;
    double* qsup = p.ws.qsup + d.qsup_off;
    for (int base = tid; base < cols * R; base += SumBatch<R>::value * kThreads) {
        constexpr int E = SumBatch<R>::value;
        const double* src[E];
        bool valid[E];
        double s[E];
#pragma unroll
        for (int e = 0; e < E; ++e) {
            const int idx = base + e * kThreads;
            valid[e] = idx < cols * R;
            const int64_t col = col0 + (valid[e] ? idx / R : 0);
            src[e] = qpart + (static_cast<int64_t>(rb0) * n + col) * R + (valid[e] ? idx % R : 0);
        }
        sums_in_order<E>(src, valid, n * R, nin, s);
#pragma unroll
        for (int e = 0; e < E; ++e) {
            const int idx = base + e * kThreads;
            if (valid[e]) qsup[(static_cast<int64_t>(sup) * n + col0 + idx / R) * R + idx % R] = s[e];
        }
    }
    if (tid == 0) *c1 = 0u;

    // 2) the last super-block of the chunk: Q_bar for the chunk's columns
    __syncthreads();
    if (tid == 0) {
        __threadfence();
        const unsigned prev = atomicAdd(&cnt[cl.b_chunk + tc.c], 1u);
        if (prev >= static_cast<unsigned>(d.nsup)) atomicOr(p.ws.status, kStatusCounter);
        s_flag = (prev == static_cast<unsigned>(d.nsup - 1));
    }
    __syncthreads();
    if (!s_flag) return;
    __threadfence();
    float* qbar = p.ws.qbar + d.qrow_off;
    float* qout = p.t.q[tc.l];
    const int r = p.r;
    const double inv_w = 1.0 / static_cast<double>(p.workers);
    for (int base = tid; base < cols * R; base += SumBatch<R>::value * kThreads) {
        constexpr int E = SumBatch<R>::value;
        const double* src[E];
        bool valid[E];
        double sums[E];
#pragma unroll
        for (int e = 0; e < E; ++e) {
            const int idx = base + e * kThreads;
            valid[e] = idx < cols * R;
            src[e] = qsup + (col0 + (valid[e] ? idx / R : 0)) * R + (valid[e] ? idx % R : 0);
        }
        sums_in_order<E>(src, valid, n * R, d.nsup, sums);
#pragma unroll
        for (int e = 0; e < E; ++e) {
            const int idx = base + e * kThreads;
            if (!valid[e]) continue;
            const int64_t col = col0 + idx / R;
            const int k = idx % R;
            const double s = sums[e];
            if (p.dist) {
                p.dist_out[d.qrow_off + col * R + k] = s;   // this rank's share of the all-reduce
                continue;
            }
            const float v = static_cast<float>(s * inv_w);
            qbar[col * R + k] = v;
            if (k < r) qout[col * r + k] = v;
        }
    }
    if (tid == 0) cnt[cl.b_chunk + tc.c] = 0u;
}

template <int R, bool SF>
__global__ void __launch_bounds__(kThreads, (R <= 8 ? 3 : 2)) k_pass_b(Params p) {
    extern __shared__ __align__(16) unsigned char smem[];
    const int t = p.tile_base + tile_index<true>();
    const int l = p.t.tile_layer[t];
    if (p.track_conv && p.iter > p.ws.conv_iter[l]) return;   // converged refresh layer
    const LayerDesc d = p.t.layers[l];
    const TileCoord tc = decode_tile(d, t, l);
    const int W = p.workers;
    const int L = p.num_layers;

    float** ep = reinterpret_cast<float**>(smem);
    float* ph_s = reinterpret_cast<float*>(smem + ((SmemB<R>::ptr_bytes(W) + 15) & ~size_t(15)));
    float* red_s = reinterpret_cast<float*>(reinterpret_cast<unsigned char*>(ph_s) +
                                            ((SmemB<R>::rows_bytes(d.tm) + 15) & ~size_t(15)));

    for (int w = threadIdx.x; w < W; w += kThreads) ep[w] = p.t.errors[w * L + l];
    load_phat_rows<R>(p, d, tc, ph_s);

    if constexpr (UseMma<R>::value) {
        if (d.vec == 4) {
            if constexpr (SF) pass_b_staged<R, SF>(p, d, tc, ep, ph_s, red_s);
            else pass_b_tc<R>(p, d, tc, ep, ph_s, reinterpret_cast<unsigned char*>(red_s));
        } else if (d.vec == 2) {
            pass_b_mma<R, 2, SF>(p, d, tc, ep, ph_s, red_s);
        } else {
            pass_b_mma<R, 1, SF>(p, d, tc, ep, ph_s, red_s);
        }
    } else {
        if (d.vec == 4) {
            if constexpr (R <= 4) pass_b_rows<R, 4, SF>(p, d, tc, ep, ph_s, red_s);
        } else if (d.vec == 2) {
            if constexpr (R <= 16) pass_b_rows<R, 2, SF>(p, d, tc, ep, ph_s, red_s);
        } else {
            pass_b_rows<R, 1, SF>(p, d, tc, ep, ph_s, red_s);
        }
    }
    pass_b_epilogue<R>(p, d, tc);
}

// P_hat = P_bar T (T = R^-1 from the orthogonalisation) for every layer,
// once per layer: float64 sums in column order over the upper-triangular T,
// rounded to float32, into the workspace (read by the second and third
// passes) and the caller's P_hat.  Grid (x, layers): layer layer_base +
// blockIdx.y, its m R elements strided over blockIdx.x; a thread's loads
// of its row are all in flight together.
template <int R>
__global__ void __launch_bounds__(kThreads) k_phat(Params p) {
    __shared__ double T_s[R * R];
    const int l = p.layer_base + static_cast<int>(blockIdx.y);
    if (p.track_conv && p.iter > p.ws.conv_iter[l]) return;   // converged refresh layer
    const LayerDesc d = p.t.layers[l];
    const double* T = p.ws.T + d.t_off;
    for (int idx = threadIdx.x; idx < R * R; idx += kThreads) T_s[idx] = T[idx];
    __syncthreads();
    const int64_t total = d.m * R;
    const double* pbar = p.ws.pbar + d.prow_off;
    float* phat = p.ws.phat + d.prow_off;
    float* out = (p.t.p_hat_out != nullptr) ? p.t.p_hat_out[l] : nullptr;
    const int r = p.r;
    for (int64_t idx = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x; idx < total;
         idx += static_cast<int64_t>(gridDim.x) * kThreads) {
        const int64_t row = idx / R;
        const int k = static_cast<int>(idx - row * R);
        const double* pr = pbar + row * R;
        double pv[R];
#pragma unroll
        for (int a = 0; a < R; ++a) pv[a] = a <= k ? __ldg(pr + a) : 0.0;
        double s = 0.0;
#pragma unroll
        for (int a = 0; a < R; ++a)
            if (a <= k) s += pv[a] * T_s[a * R + k];
        const float v = static_cast<float>(s);
        phat[idx] = v;
        if (out != nullptr && k < r) out[row * r + k] = v;
    }
}

// ---------------------------------------------------------------------------
// pass C: residual / decompression / momentum

template <int R>
struct SmemC {
    static __host__ __device__ size_t ptr_bytes(int W) { return static_cast<size_t>(W < 1 ? 1 : W) * sizeof(void*); }
    static __host__ __device__ size_t rows_bytes(int tm) { return static_cast<size_t>(tm) * R * sizeof(float); }
    static __host__ __device__ size_t wide_bytes() {
        return IsWide<R>::value ? static_cast<size_t>(R) * 4 * kWideCols * sizeof(float) : 0;
    }
    static __host__ __device__ size_t total(int W, int tm) {
        return ((ptr_bytes(W) + 15) & ~size_t(15)) + ((rows_bytes(tm) + 15) & ~size_t(15)) + wide_bytes();
    }
};

// Wide variant of the third pass (R = 16 or 32).  The tile's
// reconstruction rec = P_hat Q_bar^T (rows x chunk width) is formed once
// from shared memory (Q_bar transposed, float4 per lane) with the same
// float32 operation order as recon_dot, then applied to every worker:
// thread (warp w, lane q) owns rows w + 8 s and columns 4q .. 4q+3.
template <int R>
__device__ __forceinline__ void pass_c_wide(const Params& p, const LayerDesc& d, const TileCoord& tc,
                                            float* const* ep, const float* ph_s, float* qt_s) {
    constexpr int STR = 4 * kWideCols;
    constexpr int SR = kWideRows / kWarps;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int W = p.do_resid ? p.workers : 0;
    const int64_t n = d.n, m = d.m;
    const int64_t i0 = static_cast<int64_t>(tc.rb) * d.tm;
    const int rows = static_cast<int>(min(static_cast<int64_t>(d.tm), m - i0));
    const int64_t jc = static_cast<int64_t>(tc.c) * d.slots * d.vec;
    const int width = static_cast<int>(min(static_cast<int64_t>(d.slots) * d.vec, n - jc));
    const float* Qb = p.ws.qbar + d.qrow_off;
    for (int idx = tid; idx < R * STR; idx += kThreads) {
        const int kk = idx / STR, jj = idx % STR;
        qt_s[idx] = (jj < width) ? Qb[(jc + jj) * R + kk] : 0.f;
    }
    __syncthreads();
    // rec[s][v] = sum_k ph[row_s][k] * qbar[col_v][k], k ascending (recon_dot's
    // order); four k at a time: Q_bar for them in registers, P_hat rows as
    // float4 broadcasts, two columns per packed FMA
    float2 rec2[SR][2];
#pragma unroll
    for (int s2 = 0; s2 < SR; ++s2) rec2[s2][0] = rec2[s2][1] = make_float2(0.f, 0.f);
#pragma unroll
    for (int k4 = 0; k4 < R; k4 += 4) {
        float4 q[4];
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) q[kk] = *reinterpret_cast<const float4*>(qt_s + (k4 + kk) * STR + 4 * lane);
#pragma unroll
        for (int s2 = 0; s2 < SR; ++s2) {
            const int ii = min(warp + kWarps * s2, rows - 1);
            const float4 ph = *reinterpret_cast<const float4*>(ph_s + ii * R + k4);
            const float phk[4] = {ph.x, ph.y, ph.z, ph.w};
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const float2 pp = make_float2(phk[kk], phk[kk]);
                rec2[s2][0] = __ffma2_rn(pp, make_float2(q[kk].x, q[kk].y), rec2[s2][0]);
                rec2[s2][1] = __ffma2_rn(pp, make_float2(q[kk].z, q[kk].w), rec2[s2][1]);
            }
        }
    }
    float rec[SR][4];
#pragma unroll
    for (int s2 = 0; s2 < SR; ++s2) {
        rec[s2][0] = rec2[s2][0].x;
        rec[s2][1] = rec2[s2][0].y;
        rec[s2][2] = rec2[s2][1].x;
        rec[s2][3] = rec2[s2][1].y;
    }
    float* recon = (p.do_recon && p.t.recon_out != nullptr) ? p.t.recon_out[tc.l] : nullptr;
    float* xs = p.do_mom ? p.t.params[tc.l] : nullptr;
    float* ms = p.do_mom ? p.t.mom[tc.l] : nullptr;
    const int jq = 4 * lane;
    if (jq >= width) return;
    const bool full4 = (d.vec == 4);   // 4 columns, 16-byte aligned
    const int nv = min(4, width - jq);
#pragma unroll
    for (int s2 = 0; s2 < SR; ++s2) {
        const int ii = warp + kWarps * s2;
        if (ii >= rows) break;
        const int64_t base = (i0 + ii) * n + jc + jq;
        auto apply = [&](float* ptr, auto&& op) {
            if (full4) {
                float4 v = *reinterpret_cast<float4*>(ptr + base);
                op(v.x, 0); op(v.y, 1); op(v.z, 2); op(v.w, 3);
                *reinterpret_cast<float4*>(ptr + base) = v;
            } else {
                for (int v = 0; v < nv; ++v) op(ptr[base + v], v);
            }
        };
        if (recon != nullptr) apply(recon, [&](float& x, int v) { x = rec[s2][v]; });
        if (xs != nullptr) {
            if (full4) {
                float4 mo = *reinterpret_cast<float4*>(ms + base);
                float4 x = *reinterpret_cast<float4*>(xs + base);
                mo.x = fmaf(p.beta, mo.x, rec[s2][0]); x.x = fmaf(-p.lr, mo.x, x.x);
                mo.y = fmaf(p.beta, mo.y, rec[s2][1]); x.y = fmaf(-p.lr, mo.y, x.y);
                mo.z = fmaf(p.beta, mo.z, rec[s2][2]); x.z = fmaf(-p.lr, mo.z, x.z);
                mo.w = fmaf(p.beta, mo.w, rec[s2][3]); x.w = fmaf(-p.lr, mo.w, x.w);
                *reinterpret_cast<float4*>(ms + base) = mo;
                *reinterpret_cast<float4*>(xs + base) = x;
            } else {
                for (int v = 0; v < nv; ++v) {
                    const float mo = fmaf(p.beta, ms[base + v], rec[s2][v]);
                    ms[base + v] = mo;
                    xs[base + v] = fmaf(-p.lr, mo, xs[base + v]);
                }
            }
        }
        // E' = M - rec for every worker: a group's loads all in flight
        // before its stores (8, 4, 2, 1 workers at a time)
        auto group = [&](auto GC, int w0) {
            constexpr int G = decltype(GC)::value;
            if (full4) {
                float4 v[G];
#pragma unroll
                for (int u = 0; u < G; ++u) v[u] = *reinterpret_cast<const float4*>(ep[w0 + u] + base);
#pragma unroll
                for (int u = 0; u < G; ++u) {
                    v[u].x -= rec[s2][0];
                    v[u].y -= rec[s2][1];
                    v[u].z -= rec[s2][2];
                    v[u].w -= rec[s2][3];
                    *reinterpret_cast<float4*>(ep[w0 + u] + base) = v[u];
                }
            } else {
#pragma unroll
                for (int u = 0; u < G; ++u)
                    for (int v = 0; v < nv; ++v) ep[w0 + u][base + v] = ep[w0 + u][base + v] - rec[s2][v];
            }
        };
        int w = 0;
        for (; w + 8 <= W; w += 8) group(std::integral_constant<int, 8>{}, w);
        if (w + 4 <= W) {
            group(std::integral_constant<int, 4>{}, w);
            w += 4;
        }
        if (w + 2 <= W) {
            group(std::integral_constant<int, 2>{}, w);
            w += 2;
        }
        if (w < W) group(std::integral_constant<int, 1>{}, w);
    }
}

template <int R, int VEC>
__device__ __forceinline__ void pass_c_rows(const Params& p, const LayerDesc& d, const TileCoord& tc,
                                            float* const* ep, const float* ph_s) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int W = p.do_resid ? p.workers : 0;
    const int64_t n = d.n, m = d.m;
    const int64_t i0 = static_cast<int64_t>(tc.rb) * d.tm;
    const int64_t i1 = min(i0 + d.tm, m);
    const int s0 = tc.c * d.slots;
    const int ns = min(d.slots, d.nvec - s0);
    if (lane >= ns) return;
    const int64_t j = static_cast<int64_t>(s0 + lane) * VEC;
    constexpr int U = (VEC == 4) ? 4 : 8;

    float qb[VEC][R];
    {
        const float* Qb = p.ws.qbar + d.qrow_off;
#pragma unroll
        for (int v = 0; v < VEC; ++v)
#pragma unroll
            for (int k = 0; k < R; ++k) qb[v][k] = Qb[(j + v) * R + k];
    }
    float* recon = (p.do_recon && p.t.recon_out != nullptr) ? p.t.recon_out[tc.l] : nullptr;
    float* xs = p.do_mom ? p.t.params[tc.l] : nullptr;
    float* ms = p.do_mom ? p.t.mom[tc.l] : nullptr;

    for (int64_t i = i0 + warp; i < i1; i += kWarps) {
        float ph[R];
#pragma unroll
        for (int k = 0; k < R; ++k) ph[k] = ph_s[(i - i0) * R + k];
        float rec[VEC];
#pragma unroll
        for (int v = 0; v + 1 < VEC; v += 2) {
            const float2 r2 = recon_dot2<R>(ph, qb[v], qb[v + 1]);
            rec[v] = r2.x;
            rec[v + 1] = r2.y;
        }
        if constexpr (VEC == 1) rec[0] = recon_dot<R>(ph, qb[0]);
        const int64_t base = i * n + j;
        if (recon != nullptr) st_f32<VEC>(recon + base, rec);
        if (xs != nullptr) {
            float x[VEC], mo[VEC];
            ld_f32<VEC>(xs + base, x);
            ld_f32<VEC>(ms + base, mo);
#pragma unroll
            for (int v = 0; v < VEC; ++v) {
                mo[v] = fmaf(p.beta, mo[v], rec[v]);
                x[v] = fmaf(-p.lr, mo[v], x[v]);
            }
            st_f32<VEC>(ms + base, mo);
            st_f32<VEC>(xs + base, x);
        }
        auto group = [&](auto GC, int w0) {
            constexpr int G = decltype(GC)::value;
            float e[G][VEC];
#pragma unroll
            for (int u = 0; u < G; ++u) ld_f32<VEC>(ep[w0 + u] + base, e[u]);
#pragma unroll
            for (int u = 0; u < G; ++u) {
#pragma unroll
                for (int v = 0; v < VEC; ++v) e[u][v] = e[u][v] - rec[v];
                st_f32<VEC>(ep[w0 + u] + base, e[u]);
            }
        };
        int w = 0;
        for (; w + U <= W; w += U) group(std::integral_constant<int, U>{}, w);
        if constexpr (U > 4) {
            if (w + 4 <= W) {
                group(std::integral_constant<int, 4>{}, w);
                w += 4;
            }
        }
        if (w + 2 <= W) {
            group(std::integral_constant<int, 2>{}, w);
            w += 2;
        }
        if (w < W) group(std::integral_constant<int, 1>{}, w);
    }
}

template <int R>
__global__ void __launch_bounds__(kThreads, 2) k_pass_c(Params p) {
    extern __shared__ __align__(16) unsigned char smem[];
    const int t = p.tile_base + tile_index<false>();
    const int l = p.t.tile_layer[t];
    const LayerDesc d = p.t.layers[l];
    const TileCoord tc = decode_tile(d, t, l);
    const int W = p.workers;
    const int L = p.num_layers;
    float** ep = reinterpret_cast<float**>(smem);
    float* ph_s = reinterpret_cast<float*>(smem + ((SmemC<R>::ptr_bytes(W) + 15) & ~size_t(15)));
    float* qt_s = reinterpret_cast<float*>(reinterpret_cast<unsigned char*>(ph_s) +
                                           ((SmemC<R>::rows_bytes(d.tm) + 15) & ~size_t(15)));
    if (p.do_resid)
        for (int w = threadIdx.x; w < W; w += kThreads) ep[w] = p.t.errors[w * L + l];
    {
        const int64_t i0 = static_cast<int64_t>(tc.rb) * d.tm;
        const int rows = static_cast<int>(min(static_cast<int64_t>(d.tm), d.m - i0));
        const float* ph = p.ws.phat + d.prow_off + i0 * R;
        for (int idx = threadIdx.x; idx < rows * R; idx += kThreads) ph_s[idx] = ph[idx];
    }
    __syncthreads();
    if constexpr (IsWide<R>::value) {
        pass_c_wide<R>(p, d, tc, ep, ph_s, qt_s);
    } else {
        if (d.vec == 4) {
            if constexpr (R <= 4) pass_c_rows<R, 4>(p, d, tc, ep, ph_s);
        } else if (d.vec == 2) {
            if constexpr (R <= 16) pass_c_rows<R, 2>(p, d, tc, ep, ph_s);
        } else {
            pass_c_rows<R, 1>(p, d, tc, ep, ph_s);
        }
    }
}

// ---------------------------------------------------------------------------
// Distributed step, after the all-reduce of P: P_bar = (sum over all ranks'
// workers) / W_global, its Gram matrix (float64, pairs over warps, rows over
// lanes, fixed order) and the Cholesky factorisation into T.  One CTA per
// layer.
template <int R>
__global__ void __launch_bounds__(kThreads) k_dist_orth(Params p) {
    __shared__ double Gs[R * R];
    __shared__ double Rs[R * R];
    __shared__ double Ts[R * R];
    __shared__ int drop[R];
    const int l = blockIdx.x;
    const LayerDesc d = p.t.layers[l];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    constexpr int NG = R * (R + 1) / 2;
    double* pbar = p.ws.pbar + d.prow_off;
    const double* psum = p.dist_in + d.prow_off;
    for (int64_t idx = tid; idx < d.m * R; idx += kThreads) pbar[idx] = psum[idx] * p.inv_w_global;
    __syncthreads();
    for (int pidx = warp; pidx < NG; pidx += kWarps) {
        int a = 0, rem = pidx;
        while (rem >= R - a) {
            rem -= R - a;
            ++a;
        }
        const int b = a + rem;
        double s = 0.0;
        for (int64_t i = lane; i < d.m; i += 32) s += pbar[i * R + a] * pbar[i * R + b];
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
        if (lane == 0) {
            Gs[a * R + b] = s;
            Gs[b * R + a] = s;
        }
    }
    __syncthreads();
    if (warp == 0) {
        factor_gram_warp<R>(Gs, Rs, Ts, drop, p.r, p.drop_tol, lane);
        double* T = p.ws.T + d.t_off;
        for (int idx = lane; idx < R * R; idx += 32) T[idx] = Ts[idx];
    }
}

// Distributed step, after the all-reduce of Q: Q_bar = sum / W_global into
// the workspace (stride R) and the caller's Q (stride r).
template <int R>
__global__ void k_dist_qbar(Params p) {
    const int l = blockIdx.y;
    const LayerDesc d = p.t.layers[l];
    float* qbar = p.ws.qbar + d.qrow_off;
    float* qout = p.t.q[l];
    const double* qsum = p.dist_in + d.qrow_off;
    const int r = p.r;
    for (int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; idx < d.n * R;
         idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const float v = static_cast<float>(qsum[idx] * p.inv_w_global);
        qbar[idx] = v;
        const int k = static_cast<int>(idx % R);
        if (k < r) qout[(idx / R) * r + k] = v;
    }
}

// ---------------------------------------------------------------------------
// initial Q: Philox4x64-10 (Salmon et al., SC'11) + Box-Muller (1958)
struct Philox4x64 {
    static constexpr uint64_t M0 = 0xD2E7470EE14C6C93ull;
    static constexpr uint64_t M1 = 0xCA5A826395121157ull;
    static constexpr uint64_t W0 = 0x9E3779B97F4A7C15ull;
    static constexpr uint64_t W1 = 0xBB67AE8584CAA73Bull;
    __device__ static void run(uint64_t (&x)[4], uint64_t k0, uint64_t k1) {
#pragma unroll
        for (int rnd = 0; rnd < 10; ++rnd) {
            if (rnd) {
                k0 += W0;
                k1 += W1;
            }
            const uint64_t hi0 = __umul64hi(M0, x[0]), lo0 = M0 * x[0];
            const uint64_t hi1 = __umul64hi(M1, x[2]), lo1 = M1 * x[2];
            const uint64_t y0 = hi1 ^ x[1] ^ k0;
            const uint64_t y2 = hi0 ^ x[3] ^ k1;
            x[0] = y0;
            x[1] = lo1;
            x[2] = y2;
            x[3] = lo0;
        }
    }
};

// ---------------------------------------------------------------------------
// Rayleigh-Ritz rotation after the subspace iterations of an SVD refresh:
// C = Q_bar^T Q_bar = W diag(lambda) W^T over the block's r columns (cyclic
// Jacobi, float64, one warp, eigenvalues sorted descending, every column of
// W signed so that its largest-magnitude entry is positive); then
// P_hat W and Q_bar W, of which the first dst.r_out columns are kept.  When
// span(P_hat) holds the top left singular subspace of the worker mean, the
// kept columns are P_hat = U_r and Q_bar = V_r Sigma_r.  The source is the
// launching context's workspace (rank r = p.r, stride R); the destination
// is a context of rank dst.r_out (stride dst.RD, columns r_out..RD-1 set to
// zero) with the caller's Q and P_hat: the same context (in place, r_out =
// r) or the rank-r context an oversampled block was iterated for.  One CTA
// per layer; each row is read whole before it is written.
struct RRDst {
    const LayerDesc* layers;   // destination geometry (prow_off, qrow_off)
    float* phat;               // destination workspace rows, stride RD
    float* qbar;
    float* const* q_out;       // caller's Q, n x r_out
    float* const* p_out;       // caller's P_hat, m x r_out (table may be null, entries too)
    int RD, r_out;
};

template <int R>
__global__ void __launch_bounds__(kThreads) k_rayleigh_ritz(Params p, RRDst dst) {
    __shared__ double C[R * R];
    __shared__ double V[R * R];
    __shared__ double Wm[R * R];
    __shared__ double lam[R];
    __shared__ int order[R];
    const int l = blockIdx.x;
    const LayerDesc d = p.t.layers[l];
    const LayerDesc dd = dst.layers[l];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int r = p.r;
    constexpr int NG = R * (R + 1) / 2;
    const float* qbar = p.ws.qbar + d.qrow_off;
    const float* phat = p.ws.phat + d.prow_off;

    // 1) C = Q_bar^T Q_bar (pairs over warps, rows over lanes, fixed order)
    for (int pidx = warp; pidx < NG; pidx += kWarps) {
        int a = 0, rem = pidx;
        while (rem >= R - a) {
            rem -= R - a;
            ++a;
        }
        const int b = a + rem;
        double s = 0.0;
        for (int64_t j = lane; j < d.n; j += 32)
            s += static_cast<double>(qbar[j * R + a]) * static_cast<double>(qbar[j * R + b]);
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
        if (lane == 0) {
            C[a * R + b] = s;
            C[b * R + a] = s;
        }
    }
    __syncthreads();

    // 2) eigen-decomposition of the r x r block by cyclic Jacobi (warp 0)
    if (warp == 0) {
        for (int idx = lane; idx < R * R; idx += 32) V[idx] = (idx / R == idx % R) ? 1.0 : 0.0;
        __syncwarp();
        double scale = 0.0;
        for (int k = 0; k < r; ++k) scale += C[k * R + k] * C[k * R + k];
        for (int sweep = 0; sweep < 40; ++sweep) {
            double off = 0.0;
            for (int a = 0; a < r; ++a)
                for (int b = a + 1; b < r; ++b) off += C[a * R + b] * C[a * R + b];
            if (!(off > 1e-30 * scale)) break;   // converged (also stops on NaN)
            for (int a = 0; a < r - 1; ++a) {
                for (int b = a + 1; b < r; ++b) {
                    const double apq = C[a * R + b];
                    if (apq == 0.0) continue;
                    const double theta = (C[b * R + b] - C[a * R + a]) / (2.0 * apq);
                    const double t = (theta == 0.0) ? 1.0
                                                    : copysign(1.0, theta) / (fabs(theta) + sqrt(theta * theta + 1.0));
                    const double c = 1.0 / sqrt(t * t + 1.0);
                    const double sn = t * c;
                    const int k = lane;
                    if (k < r) {
                        const double cp = C[k * R + a], cq = C[k * R + b];
                        C[k * R + a] = c * cp - sn * cq;
                        C[k * R + b] = sn * cp + c * cq;
                    }
                    __syncwarp();
                    if (k < r) {
                        const double rp = C[a * R + k], rq = C[b * R + k];
                        C[a * R + k] = c * rp - sn * rq;
                        C[b * R + k] = sn * rp + c * rq;
                        const double vp = V[k * R + a], vq = V[k * R + b];
                        V[k * R + a] = c * vp - sn * vq;
                        V[k * R + b] = sn * vp + c * vq;
                    }
                    __syncwarp();
                }
            }
        }
        if (lane == 0) {
            for (int k = 0; k < R; ++k) {
                lam[k] = (k < r) ? C[k * R + k] : 0.0;
                order[k] = k;
            }
            for (int a = 0; a < r; ++a) {   // selection sort, descending, stable
                int best = a;
                for (int b = a + 1; b < r; ++b)
                    if (lam[order[b]] > lam[order[best]]) best = b;
                const int tmp = order[best];
                for (int b = best; b > a; --b) order[b] = order[b - 1];
                order[a] = tmp;
            }
        }
        __syncwarp();
        for (int idx = lane; idx < R * R; idx += 32) Wm[idx] = 0.0;
        __syncwarp();
        if (lane < r) {
            const int src = order[lane];
            int arg = 0;
            double best = -1.0;
            for (int k = 0; k < r; ++k) {
                const double v = fabs(V[k * R + src]);
                if (v > best) {
                    best = v;
                    arg = k;
                }
            }
            const double sg = (V[arg * R + src] < 0.0) ? -1.0 : 1.0;
            for (int k = 0; k < r; ++k) Wm[k * R + lane] = sg * V[k * R + src];
        }
    }
    __syncthreads();

    // 3) rotate Q_bar and P_hat (one row per thread), keep r_out columns
    const int RD = dst.RD, ro = dst.r_out;
    float* qd = dst.qbar + dd.qrow_off;
    float* pd = dst.phat + dd.prow_off;
    float* qout = dst.q_out[l];
    float* pout = (dst.p_out != nullptr) ? dst.p_out[l] : nullptr;
    auto rotate_rows = [&](const float* src, float* dws, float* out, int64_t rows) {
        for (int64_t j = tid; j < rows; j += kThreads) {
            double row[R];
#pragma unroll
            for (int k = 0; k < R; ++k) row[k] = src[j * R + k];
            for (int k = 0; k < RD; ++k) {
                double v = 0.0;
                if (k < ro) {
#pragma unroll
                    for (int a = 0; a < R; ++a) v += row[a] * Wm[a * R + k];
                }
                const float f = static_cast<float>(v);
                dws[j * RD + k] = f;
                if (out != nullptr && k < ro) out[j * ro + k] = f;
            }
        }
    };
    rotate_rows(qbar, qd, qout, d.n);
    rotate_rows(phat, pd, pout, d.m);
}

// Q block of an oversampled refresh: the caller's warm start Q (n x r) in
// the first r columns, fresh N(0, 1) draws in the other rp - r (the
// k_init_q generator: Philox4x64-10 keyed by (seed, l), counter
// (b, draw, 0, 0) for block b = e / 4 of the extra elements
// e = j * (rp - r) + (k - r), Box-Muller in float64).
__global__ void k_assemble_q(float* const* qdst, float* const* qsrc, const LayerDesc* layers, int r, int rp,
                             uint64_t seed, uint64_t draw) {
    const int l = blockIdx.y;
    const int64_t n = layers[l].n;
    const int px = rp - r;
    float* out = qdst[l];
    const float* in = qsrc[l];
    const int64_t t0 = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t e = t0; e < n * r; e += stride) out[(e / r) * rp + e % r] = in[e];
    const int64_t total = n * px;
    constexpr double kTwoPi = 2.0 * 3.141592653589793;
    for (int64_t b = t0; b < (total + 3) / 4; b += stride) {
        uint64_t x[4] = {static_cast<uint64_t>(b), draw, 0ull, 0ull};
        Philox4x64::run(x, seed, static_cast<uint64_t>(l));
        double z[4];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const double u0 = (static_cast<double>(x[2 * h] >> 11) + 0.5) * (1.0 / 9007199254740992.0);
            const double u1 = (static_cast<double>(x[2 * h + 1] >> 11) + 0.5) * (1.0 / 9007199254740992.0);
            const double rho = sqrt(-2.0 * log(u0));
            z[2 * h] = rho * cos(kTwoPi * u1);
            z[2 * h + 1] = rho * sin(kTwoPi * u1);
        }
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            const int64_t e = 4 * b + t;
            if (e < total) out[(e / px) * rp + r + e % px] = static_cast<float>(z[t]);
        }
    }
}

// ---------------------------------------------------------------------------
// small tensors: mean over workers (+ optional momentum)
__global__ void k_vec_mean(const float* const* vecs, float* const* out, const int64_t* len, int count, int W,
                           float inv_w, float* const* params, float* const* mom, float lr, float beta) {
    const int k = blockIdx.y;
    const int64_t nk = len[k];
    float* o = out[k];
    float* x = (params != nullptr) ? params[k] : nullptr;
    float* mo = (mom != nullptr) ? mom[k] : nullptr;
    for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < nk;
         e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        // workers summed in order; eight workers' loads in flight at a time
        float s = 0.f;
        int w = 0;
        for (; w + 8 <= W; w += 8) {
            float v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) v[u] = vecs[(w + u) * count + k][e];
#pragma unroll
            for (int u = 0; u < 8; ++u) s += v[u];
        }
        for (; w < W; ++w) s += vecs[w * count + k][e];
        const float g = s * inv_w;
        o[e] = g;
        if (x != nullptr && mo != nullptr) {
            const float mv = fmaf(beta, mo[e], g);
            mo[e] = mv;
            x[e] = fmaf(-lr, mv, x[e]);
        }
    }
}

__global__ void k_init_q(float* const* q, const LayerDesc* layers, int r, uint64_t seed, uint64_t draw) {
    const int l = blockIdx.y;
    const int64_t total = layers[l].n * r;
    const int64_t nb = (total + 3) / 4;
    float* out = q[l];
    constexpr double kTwoPi = 2.0 * 3.141592653589793;
    for (int64_t b = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; b < nb;
         b += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        uint64_t x[4] = {static_cast<uint64_t>(b), draw, 0ull, 0ull};
        Philox4x64::run(x, seed, static_cast<uint64_t>(l));
        double z[4];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const double u0 = (static_cast<double>(x[2 * h] >> 11) + 0.5) * (1.0 / 9007199254740992.0);
            const double u1 = (static_cast<double>(x[2 * h + 1] >> 11) + 0.5) * (1.0 / 9007199254740992.0);
            const double rho = sqrt(-2.0 * log(u0));
            z[2 * h] = rho * cos(kTwoPi * u1);
            z[2 * h + 1] = rho * sin(kTwoPi * u1);
        }
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            const int64_t e = 4 * b + t;
            if (e < total) out[e] = static_cast<float>(z[t]);
        }
    }
}

}  // namespace psgd
