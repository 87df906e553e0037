// Device-side types and helpers shared by the PowerSGD kernels.
#pragma once

#include <cstdint>
#include <type_traits>
#include <cuda_runtime.h>

namespace psgd {

constexpr int kThreads = 256;          // threads per CTA in every streaming kernel
constexpr int kWarps = kThreads / 32;
constexpr int kMaxWorkers = 256;
constexpr int kMaxRank = 32;
constexpr int kRowsFloatsMax = 4096;   // tile rows x R bound (the second pass's P_hat rows)

// Per-layer geometry and workspace offsets (element counts), built on the
// host at context creation.  A "tile" is TM rows x one column chunk of a
// layer, for all W workers; a chunk is at most 32 vector slots of VEC
// columns (one slot per lane).
struct LayerDesc {
    int64_t m, n;
    int vec;        // columns per lane load (4, 2 or 1)
    int nvec;       // n / vec
    int nchunk;     // column chunks
    int slots;      // vector slots per chunk (<= 32); chunks are balanced
    int tm;         // rows per tile (multiple of 8)
    int nrb;        // row blocks = ceil(m / tm)
    int nsup;       // super-blocks of kSuper row blocks (two-level reductions)
    int pad_;
    int64_t tile_begin;  // index of this layer's first tile in the grouped grid
    int64_t prow_off;    // P_bar (double) / P_hat (float) rows, stride R
    int64_t qrow_off;    // Q_bar rows (stride R floats)
    int64_t ppart_off;   // P partials [nchunk][m][R] doubles
    int64_t qpart_off;   // Q partials [nrb][n][R] doubles
    int64_t gram_off;    // Gram partials [nrb][R(R+1)/2] doubles
    int64_t gsup_off;    // Gram super-block partials [nsup][R(R+1)/2] doubles
    int64_t qsup_off;    // Q super-block partials [nsup][n][R] doubles
    int64_t t_off;       // T = R^-1, R x R doubles
    int64_t cnt_off;     // counters, see counter_layout()
};

// Row-block partials are summed in two levels: every kSuper row blocks into
// a super-block partial (by the last of them to finish), then the
// super-blocks (by the last super-block).  Both levels sum in index order.
constexpr int kSuper = 32;

// Counter offsets inside a layer's counter block.
struct CounterLayout {
    int64_t a_rb, a_sup, a_layer, b_sup, b_chunk, total;
};
__host__ __device__ inline CounterLayout counter_layout(int nrb, int nsup, int nchunk) {
    CounterLayout c;
    c.a_rb = 0;                                   // [nrb]  chunk tiles done per row block (pass A)
    c.a_sup = nrb;                                // [nsup] row blocks done per super-block (pass A)
    c.a_layer = nrb + nsup;                       // [1]    super-blocks done (pass A)
    c.b_sup = c.a_layer + 1;                      // [nchunk][nsup] row-block tiles done (pass B)
    c.b_chunk = c.b_sup + static_cast<int64_t>(nchunk) * nsup;  // [nchunk] super-blocks done (pass B)
    c.total = c.b_chunk + nchunk;
    return c;
}

struct Tables {
    const LayerDesc* layers;
    const int* tile_layer;        // tile -> layer
    const void* const* grads;     // [W*L]
    float* const* errors;         // [W*L]
    float* const* q;              // [L] caller's Q state (n x r)
    float* const* p_hat_out;      // [L] entries may be null
    float* const* recon_out;      // [L] entries may be null
    float* const* params;         // [L] momentum targets
    float* const* mom;            // [L]
};

// Accuracy: products are summed in float32 only over short runs (one
// worker's VEC columns in pass A, one tile's rows in pass B); every longer
// sum (lanes, chunks, warps, row blocks) and P_bar itself are float64.
// The weak columns of P_hat (directions near the noise floor) amplify the
// rounding error of P_bar by ||pbar_j|| / ||pbar_j after projection||.
struct Work {
    double* pbar;
    float* phat;
    float* qbar;
    double* ppart;
    double* qpart;
    double* gram;
    double* gsup;
    double* qsup;
    double* T;
    unsigned* cnt;
    int* status;
    // SVD refresh with oversampling: the iteration after which each layer
    // stops (set by the first pass once its convergence bound is met)
    int* conv_iter;
};

struct Params {
    Tables t;
    Work ws;
    int num_layers, workers, r;
    float inv_w;
    float lr, beta;
    double drop_tol;
    int use_prev;   // lazy first pass: rebuild E' from the previous P_hat, Q_bar
    int do_recon, do_mom, do_resid;
    // distributed step: the first two passes stop at this rank's partial
    // sums (rows of P, rows of Q, not divided by the worker count), written
    // to dist_out; the all-reduced sums come back through dist_in.
    int dist;
    double* dist_out;
    const double* dist_in;
    double inv_w_global;
    // subspace iterations of an SVD refresh: this launch's iteration number
    // (1, 2, ...); with track_conv, layers whose conv_iter is below it are
    // skipped, and the first pass's factorisation sets conv_iter once
    // (lambda_{r'} / lambda_{r_conv})^(iter - 1) <= conv_eps
    int iter, track_conv, r_conv;
    double conv_eps;
    // testing the bounded waits: the tensor-core second pass issues no
    // products (and commits none), so its waits run out
    int stall_products;
    // a launch over a range of layers (host-buffer steps overlap the upload
    // of later layers with the passes of earlier ones): the first tile of
    // the grouped passes' grids and the first layer of the P_hat grid
    int tile_base, layer_base;
};

enum : int {
    kStatusCounter = 1,   // a reduction counter held an impossible value
    kStatusTimeout = 2    // a bounded wait on the tensor cores ran out (about one second)
};

// ---- loads and stores ------------------------------------------------------

// bf16 -> f32 is exact: the bf16 bits are the top half of the f32 bits.
__device__ __forceinline__ float bf16_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }

template <int VEC>
__device__ __forceinline__ void ld_f32(const float* p, float (&x)[VEC]) {
    if constexpr (VEC == 4) {
        const float4 t = *reinterpret_cast<const float4*>(p);
        x[0] = t.x; x[1] = t.y; x[2] = t.z; x[3] = t.w;
    } else if constexpr (VEC == 2) {
        const float2 t = *reinterpret_cast<const float2*>(p);
        x[0] = t.x; x[1] = t.y;
    } else {
        x[0] = *p;
    }
}

template <int VEC>
__device__ __forceinline__ void st_f32(float* p, const float (&x)[VEC]) {
    if constexpr (VEC == 4) {
        *reinterpret_cast<float4*>(p) = make_float4(x[0], x[1], x[2], x[3]);
    } else if constexpr (VEC == 2) {
        *reinterpret_cast<float2*>(p) = make_float2(x[0], x[1]);
    } else {
        *p = x[0];
    }
}

// Gradients are read once per step: streaming (evict-first) loads.
template <typename GT, int VEC>
__device__ __forceinline__ void ld_grad(const GT* p, float (&x)[VEC]);

template <>
__device__ __forceinline__ void ld_grad<float, 4>(const float* p, float (&x)[4]) {
    const float4 t = __ldcs(reinterpret_cast<const float4*>(p));
    x[0] = t.x; x[1] = t.y; x[2] = t.z; x[3] = t.w;
}
template <>
__device__ __forceinline__ void ld_grad<float, 2>(const float* p, float (&x)[2]) {
    const float2 t = __ldcs(reinterpret_cast<const float2*>(p));
    x[0] = t.x; x[1] = t.y;
}
template <>
__device__ __forceinline__ void ld_grad<float, 1>(const float* p, float (&x)[1]) {
    x[0] = __ldcs(p);
}
template <>
__device__ __forceinline__ void ld_grad<uint16_t, 4>(const uint16_t* p, float (&x)[4]) {
    const uint2 t = __ldcs(reinterpret_cast<const uint2*>(p));
    x[0] = bf16_lo(t.x); x[1] = bf16_hi(t.x); x[2] = bf16_lo(t.y); x[3] = bf16_hi(t.y);
}
template <>
__device__ __forceinline__ void ld_grad<uint16_t, 2>(const uint16_t* p, float (&x)[2]) {
    const unsigned int t = __ldcs(reinterpret_cast<const unsigned int*>(p));
    x[0] = bf16_lo(t); x[1] = bf16_hi(t);
}
template <>
__device__ __forceinline__ void ld_grad<uint16_t, 1>(const uint16_t* p, float (&x)[1]) {
    const unsigned short t = __ldcs(reinterpret_cast<const unsigned short*>(p));
    x[0] = __uint_as_float(static_cast<uint32_t>(t) << 16);
}

// ---- warp reductions -------------------------------------------------------

// Transposing butterfly: N partial values per lane (N a power of two,
// N <= 32) are summed over the 32 lanes with N-1 + (5 - log2 N) shuffles.
// Afterwards v[0] of lane L holds the full sum of value index
// L >> (5 - log2 N); every lane of that group of 32/N lanes holds it.
// The pattern is fixed, so the summation order is deterministic.
template <typename T, int CNT, int OFF>
struct TransposeReduce {
    __device__ __forceinline__ static void run(T* v, int lane) {
        if constexpr (OFF >= 1) {
            if constexpr (CNT > 1) {
                constexpr int H = CNT / 2;
                const bool upper = (lane & OFF) != 0;
#pragma unroll
                for (int i = 0; i < H; ++i) {
                    const T send = upper ? v[i] : v[i + H];
                    const T keep = upper ? v[i + H] : v[i];
                    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, OFF);
                }
                TransposeReduce<T, H, OFF / 2>::run(v, lane);
            } else {
                v[0] += __shfl_xor_sync(0xffffffffu, v[0], OFF);
                TransposeReduce<T, 1, OFF / 2>::run(v, lane);
            }
        }
    }
};

template <int N>
struct Log2 { static constexpr int value = 1 + Log2<N / 2>::value; };
template <>
struct Log2<1> { static constexpr int value = 0; };

// acc[k] = fma(a, x[k], acc[k]) for k < R, two k per packed fp32x2 FMA
// (each component rounds exactly like fmaf)
template <int R>
__device__ __forceinline__ void axpy(float* acc, float a, const float* x) {
    if constexpr (R >= 2) {
        const float2 aa = make_float2(a, a);
#pragma unroll
        for (int k = 0; k < R; k += 2) {
            const float2 r = __ffma2_rn(aa, make_float2(x[k], x[k + 1]), make_float2(acc[k], acc[k + 1]));
            acc[k] = r.x;
            acc[k + 1] = r.y;
        }
    } else {
        acc[0] = fmaf(a, x[0], acc[0]);
    }
}

// reconstruction of one element: sum_k ph[k] * qb[k], fixed order
template <int R>
__device__ __forceinline__ float recon_dot(const float (&ph)[R], const float* qb) {
    float s = 0.f;
#pragma unroll
    for (int k = 0; k < R; ++k) s = fmaf(ph[k], qb[k], s);
    return s;
}

// recon_dot for two elements at once (same per-element operation order)
template <int R>
__device__ __forceinline__ float2 recon_dot2(const float (&ph)[R], const float* qb0, const float* qb1) {
    float2 s = make_float2(0.f, 0.f);
#pragma unroll
    for (int k = 0; k < R; ++k) s = __ffma2_rn(make_float2(ph[k], ph[k]), make_float2(qb0[k], qb1[k]), s);
    return s;
}

}  // namespace psgd
