// YOCO++ residual KV composition fused with the cache append.
//
// YOCO++: Enhancing YOCO with KV Residual Connections, section 2 ("method"):
// for a self-decoder layer i in {2..L/2} the cached keys/values are
//   K'_i = lambda (aK1 K_1 + aK2 K_i),   V'_i = lambda (aV1 V_1 + aV2 V_i),
// and (key innovation 1, cache strategy) the composed values are what is
// stored, so decoding later reads one KV set per layer.
//
// The kernel is a pure HBM stream: per (token, head) row it reads four input
// rows and writes two cache rows.  Each thread moves 16-byte chunks with
// 128-bit loads (read-once, no L1 allocation) and stores 128 bits, in a
// grid-stride loop over a grid of one 1024-thread CTA per SM.
//
// Arithmetic.  The weighted sum a1*x1 + a2*xi can cancel almost completely
// (x1, xi ~ N(0,1) and |a1| ~ |a2|), and a plain fp32 evaluation then loses
// the low bits that decide the stored bf16 value.  So the inner sum is formed
// with error-free transformations: each product as an unevaluated pair
// p + e via one FMA (TwoProduct, Ogita, Rump and Oishi, "Accurate sum and
// dot product", SIAM J. Sci. Comput. 2005), the two leading parts added with
// Knuth's TwoSum (The Art of Computer Programming, vol. 2, 4.2.2), and the
// small parts folded in; lambda is applied last, as in the equations.  The
// fp32 result is then within a few fp32 roundings of the exact value relative
// to the value itself, and is rounded once to the cache type.
#pragma once

#include "common.cuh"

namespace yocopp {

struct ComposeParams {
    const uint8_t* k1;
    const uint8_t* v1;
    const uint8_t* ki;
    const uint8_t* vi;
    uint8_t* ck;
    uint8_t* cv;
    const int32_t* block_table;  // nullptr: contiguous cache
    const int32_t* pos;
    const int32_t* cu_new;       // nullptr: uniform n per sequence
    float ak1, ak2, av1, av2, lam;  // residual weights and scale, as given
    int64_t total_rows;          // input rows x kv heads
    int32_t hkv, batch, n_uniform, capacity, block_size, mbps, num_blocks;
};

// lambda * (a1 * x1 + a2 * xi) for two lanes; na1 = -a1, na2 = -a2.
__device__ __forceinline__ float2 compose2(float2 x1, float2 xi, float2 na1, float2 na2, float2 a1, float2 a2,
                                           float2 lam) {
    const float2 p1 = fmul2(a1, x1);
    const float2 n1 = ffma2(na1, x1, p1);          // p1 - a1*x1, exact
    const float2 p2 = fmul2(a2, xi);
    const float2 n2 = ffma2(na2, xi, p2);          // p2 - a2*xi, exact
    const float2 s = fadd2(p1, p2);                // TwoSum(p1, p2) = s + err, exact
    const float2 bb = fsub2(s, p1);
    const float2 err = fadd2(fsub2(p1, fsub2(s, bb)), fsub2(p2, bb));
    const float2 lo = fsub2(err, fadd2(n1, n2));   // a1*x1 + a2*xi = s + lo (to ~2^-48 of the terms)
    return ffma2(lam, s, fmul2(lam, lo));
}

// Rounding to bf16.  The fp32 value y from compose2 is within about one fp32
// ulp of the exact composition, so converting it (nearest, ties to even)
// rounds as the exact value does unless y lies within a few fp32 ulps of a
// bf16 rounding midpoint: rounding to fp32 can carry a value onto a midpoint,
// or (with the few-ulp slack) just past it.  Those values, about 5 in 2^16,
// take the slow path: the composition in fp64, evaluated as written (inner
// weighted sum, then lambda), rounded once to bf16.  The fp64 -> bf16 rounding
// goes through fp32 with round-to-odd, which keeps a single rounding because
// fp32 carries more than two extra bits (Boldo and Melquiond, "When double
// rounding is odd", 2005).
__device__ __forceinline__ bool near_bf16_midpoint(float y) {
    return ((__float_as_uint(y) - 0x7FFEu) & 0xFFFFu) <= 4u;
}

__device__ __forceinline__ float f64_to_f32_round_odd(double v) {
    float r;
    asm("cvt.rz.f32.f64 %0, %1;" : "=f"(r) : "d"(v));
    if (double(r) != v) r = __uint_as_float(__float_as_uint(r) | 1u);
    return r;
}

__device__ __noinline__ uint32_t compose2_bf16_exact(float2 x1, float2 xi, float a1, float a2, float lam) {
    const double ex = __dmul_rn(double(lam), __dadd_rn(__dmul_rn(double(a1), double(x1.x)),
                                                        __dmul_rn(double(a2), double(xi.x))));
    const double ey = __dmul_rn(double(lam), __dadd_rn(__dmul_rn(double(a1), double(x1.y)),
                                                        __dmul_rn(double(a2), double(xi.y))));
    return float2_to_bf16x2(f64_to_f32_round_odd(ex), f64_to_f32_round_odd(ey));
}

struct ComposeCoef {
    float2 a1, a2, na1, na2, lam;
};

__device__ __forceinline__ ComposeCoef make_coef(float a1, float a2, float lam) {
    ComposeCoef c;
    c.a1 = make_float2(a1, a1);
    c.a2 = make_float2(a2, a2);
    c.na1 = make_float2(-a1, -a1);
    c.na2 = make_float2(-a2, -a2);
    c.lam = make_float2(lam, lam);
    return c;
}

// Compose one 16-byte chunk and round once to the cache type.
template <typename T>
__device__ __forceinline__ uint4 compose_chunk(uint4 a1, uint4 ai, const ComposeCoef& c);

template <>
__device__ __forceinline__ uint4 compose_chunk<__nv_bfloat16>(uint4 a1, uint4 ai, const ComposeCoef& c) {
    const uint32_t* w1 = reinterpret_cast<const uint32_t*>(&a1);
    const uint32_t* wi = reinterpret_cast<const uint32_t*>(&ai);
    uint4 r;
    uint32_t* wr = reinterpret_cast<uint32_t*>(&r);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const float2 x1 = bf16x2_to_float2(w1[k]), xi = bf16x2_to_float2(wi[k]);
        const float2 y = compose2(x1, xi, c.na1, c.na2, c.a1, c.a2, c.lam);
        uint32_t w = float2_to_bf16x2(y.x, y.y);
        if (near_bf16_midpoint(y.x) | near_bf16_midpoint(y.y))
            w = compose2_bf16_exact(x1, xi, c.a1.x, c.a2.x, c.lam.x);
        wr[k] = w;
    }
    return r;
}

template <>
__device__ __forceinline__ uint4 compose_chunk<float>(uint4 a1, uint4 ai, const ComposeCoef& c) {
    const float2* f1 = reinterpret_cast<const float2*>(&a1);
    const float2* fi = reinterpret_cast<const float2*>(&ai);
    uint4 r;
    float2* fr = reinterpret_cast<float2*>(&r);
#pragma unroll
    for (int k = 0; k < 2; ++k) fr[k] = compose2(f1[k], fi[k], c.na1, c.na2, c.a1, c.a2, c.lam);
    return r;
}

// Cache byte offset of (sequence b, new-token index j, head h), or -1 if the
// position or its block is out of range (recorded in the device status).
template <int ROWB>
__device__ __forceinline__ int64_t cache_row_offset(const ComposeParams& p, int b, int j, int h) {
    const int position = __ldg(p.pos + b) + j;
    if (position < 0 || position >= p.capacity) {
        record_status(YOCOPP_ECAPACITY);
        return -1;
    }
    if (p.block_table == nullptr)
        return ((int64_t(b) * p.hkv + h) * p.capacity + position) * ROWB;
    const int blk = __ldg(p.block_table + int64_t(b) * p.mbps + position / p.block_size);
    if (blk < 0 || blk >= p.num_blocks) {
        record_status(YOCOPP_EDEVICE_CHECK);
        return -1;
    }
    return ((int64_t(blk) * p.hkv + h) * p.block_size + position % p.block_size) * ROWB;
}

// Launch shape (compile-time; the defaults are the measured best on B200).
// One 1024-thread CTA per SM, two chunks of every stream in flight per thread
// (measured +3% over one at 32 x 8192, the same on the ragged paged batch): the
// grid is exactly resident (no second-wave tail), and each iteration of the
// grid-stride loop sweeps 2 x 148 x 1024 consecutive chunks of every stream.
#ifndef YOCOPP_COMPOSE_THREADS
#define YOCOPP_COMPOSE_THREADS 1024
#endif
#ifndef YOCOPP_COMPOSE_UNROLL
#define YOCOPP_COMPOSE_UNROLL 2
#endif
#ifndef YOCOPP_COMPOSE_CTAS_PER_SM
#define YOCOPP_COMPOSE_CTAS_PER_SM 1
#endif

template <typename T, int ROWB>
__global__ void __launch_bounds__(YOCOPP_COMPOSE_THREADS) compose_append_kernel(ComposeParams p) {
    constexpr int CPR = ROWB / 16;                 // 16-byte chunks per (token, head) row
    constexpr int U = YOCOPP_COMPOSE_UNROLL;       // chunks in flight per thread
    extern __shared__ int s_cu[];   // staged prefix offsets (ragged batches only)

    if (p.cu_new != nullptr) {
        for (int i = threadIdx.x; i <= p.batch; i += blockDim.x) s_cu[i] = p.cu_new[i];
        __syncthreads();
    }
    const int64_t nchunks = p.total_rows * CPR;
    const int64_t stride = int64_t(gridDim.x) * blockDim.x;
    const ComposeCoef ck = make_coef(p.ak1, p.ak2, p.lam);
    const ComposeCoef cv = make_coef(p.av1, p.av2, p.lam);
    // (token, head) rows fit 32 bits for every workload the host accepts below 2^31 rows: the
    // row -> (token, head, sequence) arithmetic then runs in 32-bit integer division
    const bool narrow = p.total_rows < (int64_t(1) << 31);
    int bc = 0;  // ragged batches: this thread's last sequence (its chunks only move forward)

    for (int64_t i0 = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i0 < nchunks; i0 += stride * U) {
        uint4 x1k[U], xik[U], x1v[U], xiv[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t idx = i0 + u * stride;
            if (idx < nchunks) {
                const int64_t off = (idx / CPR) * ROWB + (idx % CPR) * 16;
                x1k[u] = ld_stream(p.k1 + off);
                xik[u] = ld_stream(p.ki + off);
                x1v[u] = ld_stream(p.v1 + off);
                xiv[u] = ld_stream(p.vi + off);
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t idx = i0 + u * stride;
            if (idx >= nchunks) continue;
            const int64_t row = idx / CPR;
            const int c = int(idx % CPR);
            int64_t tok;
            int h;
            if (narrow) {
                const uint32_t r32 = uint32_t(row), hk = uint32_t(p.hkv);
                tok = int64_t(r32 / hk);
                h = int(r32 - uint32_t(tok) * hk);
            } else {
                tok = row / p.hkv;
                h = int(row % p.hkv);
            }
            int b, j;
            if (p.cu_new == nullptr) {
                if (narrow) {
                    b = int(uint32_t(tok) / uint32_t(p.n_uniform));
                } else {
                    b = int(tok / p.n_uniform);
                }
                j = int(tok - int64_t(b) * p.n_uniform);
            } else {
                // largest b with s_cu[b] <= tok (skips empty sequences): a few steps on from this
                // thread's last sequence, else a binary search
                if (tok < s_cu[bc]) bc = 0;
                int steps = 0;
                while (bc + 1 < p.batch && s_cu[bc + 1] <= tok && steps < 4) {
                    ++bc;
                    ++steps;
                }
                if (bc + 1 < p.batch && s_cu[bc + 1] <= tok) {
                    int lo = bc, hi = p.batch;  // invariant: s_cu[lo] <= tok < s_cu[hi]
                    while (hi - lo > 1) {
                        const int mid = (lo + hi) >> 1;
                        if (s_cu[mid] <= tok) lo = mid; else hi = mid;
                    }
                    bc = lo;
                }
                b = bc;
                j = int(tok - s_cu[b]);
            }
            const int64_t dst = cache_row_offset<ROWB>(p, b, j, h);
            if (dst < 0) continue;
            st_global(p.ck + dst + c * 16, compose_chunk<T>(x1k[u], xik[u], ck));
            st_global(p.cv + dst + c * 16, compose_chunk<T>(x1v[u], xiv[u], cv));
        }
    }
}

}  // namespace yocopp
