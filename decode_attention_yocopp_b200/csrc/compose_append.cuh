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
// the low bits that decide the stored bf16 value.  So each product is formed
// as an unevaluated pair p - n whose error n comes from one FMA, exactly
// (TwoProduct, Ogita, Rump and Oishi, "Accurate sum and dot product", SIAM J.
// Sci. Comput. 2005); the leading parts are added in fp32, s = fl(p1 + p2),
// the errors folded in, and lambda applied last, as in the equations:
//   y = fl(lambda s - fl(lambda fl(n1 + n2))).
// Where the sum cancels (p1, p2 of opposite signs within a factor 2) s is
// exact (Sterbenz), and otherwise its rounding error is at most u |s|
// (u = 2^-24) with |s| close to the result, so |y - lambda (a1 x1 + a2 xi)|
// stays below about 2 u |y| + u^2 lambda (|p1| + |p2|): under two fp32 ulps
// of y unless the sum cancels to ~2^-40 of its terms.  y is then rounded once
// to the cache type.
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
    // n / d for n < 2^31 by multiply-high and shift (fast_div), for d = hkv and n_uniform;
    // log2 of the (power-of-two) block size
    uint32_t hkv_m, hkv_s, nu_m, nu_s;
    int32_t bs_log2;
};

// Division by an invariant divisor d through a multiply-high (Granlund and
// Montgomery, "Division by invariant integers using multiplication", PLDI
// 1994, round-up variant): with l = ceil(log2 d) and m = ceil(2^(31+l) / d),
// floor(n m / 2^(31+l)) = floor(n / d) for every 0 <= n < 2^31, because
// m = 2^(31+l)/d + e with 0 <= e < 1 adds n e / 2^(31+l) < 2^-l <= 1/d to
// n / d, less than the distance to the next integer.  m < 2^32 for d >= 2;
// m = 0 stands for d = 1.
struct FastDiv {
    uint32_t m, s;  // s = l - 1
};
inline FastDiv make_fast_div(uint32_t d) {
    if (d <= 1) return FastDiv{0u, 0u};
    uint32_t l = 0;
    while ((uint64_t(1) << l) < d) ++l;
    const uint64_t m = ((uint64_t(1) << (31 + l)) + d - 1) / d;
    return FastDiv{uint32_t(m), l - 1};
}
__device__ __forceinline__ uint32_t fast_div(uint32_t n, uint32_t m, uint32_t s) {
    return m != 0u ? (__umulhi(n, m) >> s) : n;
}

// lambda * (a1 * x1 + a2 * xi) for two lanes; na1 = -a1, na2 = -a2, nlam = -lambda.
__device__ __forceinline__ float2 compose2(float2 x1, float2 xi, float2 na1, float2 na2, float2 a1, float2 a2,
                                           float2 lam, float2 nlam) {
    const float2 p1 = fmul2(a1, x1);
    const float2 n1 = ffma2(na1, x1, p1);          // p1 - a1*x1, exact
    const float2 p2 = fmul2(a2, xi);
    const float2 n2 = ffma2(na2, xi, p2);          // p2 - a2*xi, exact
    const float2 s = fadd2(p1, p2);                // a1*x1 + a2*xi = s + (p1 + p2 - s) - (n1 + n2)
    return ffma2(lam, s, fmul2(nlam, fadd2(n1, n2)));
}

// Rounding to bf16.  The fp32 value y from compose2 is within two fp32 ulps
// of the exact composition, so converting it (nearest, ties to even) rounds as
// the exact value does unless y lies within a few fp32 ulps of a bf16
// rounding midpoint.  Those values, whose low 16 bits lie within 3 of the
// midpoint's (0x8000), about 7 in 2^16, take the slow path: the composition
// in fp64, evaluated as written (inner weighted sum, then lambda), rounded
// once to bf16.  A y outside the window is 4 or more ulps from the midpoint,
// more than the error, so the exact value lies on its side.  The fp64 -> bf16 rounding
// goes through fp32 with round-to-odd, which keeps a single rounding because
// fp32 carries more than two extra bits (Boldo and Melquiond, "When double
// rounding is odd", 2005).
__device__ __forceinline__ bool near_bf16_midpoint(float y) {
    return ((__float_as_uint(y) - 0x7FFDu) & 0xFFFFu) <= 6u;
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
    float2 a1, a2, na1, na2, lam, nlam;
};

__device__ __forceinline__ ComposeCoef make_coef(float a1, float a2, float lam) {
    ComposeCoef c;
    c.a1 = make_float2(a1, a1);
    c.a2 = make_float2(a2, a2);
    c.na1 = make_float2(-a1, -a1);
    c.na2 = make_float2(-a2, -a2);
    c.lam = make_float2(lam, lam);
    c.nlam = make_float2(-lam, -lam);
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
        const float2 y = compose2(x1, xi, c.na1, c.na2, c.a1, c.a2, c.lam, c.nlam);
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
    for (int k = 0; k < 2; ++k) fr[k] = compose2(f1[k], fi[k], c.na1, c.na2, c.a1, c.a2, c.lam, c.nlam);
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
// One 1024-thread CTA per SM, one chunk of every stream in flight per thread:
// the grid is exactly resident (no second-wave tail), and each iteration of the
// grid-stride loop sweeps 148 x 1024 consecutive chunks of every stream.  Two
// chunks per thread (58 registers) measured 5% slower at 32 x 8192, more
// resident threads (1536 per SM, 40 registers) 7% slower.
#ifndef YOCOPP_COMPOSE_THREADS
#define YOCOPP_COMPOSE_THREADS 1024
#endif
#ifndef YOCOPP_COMPOSE_UNROLL
#define YOCOPP_COMPOSE_UNROLL 1
#endif
#ifndef YOCOPP_COMPOSE_CTAS_PER_SM
#define YOCOPP_COMPOSE_CTAS_PER_SM 1
#endif

template <typename T, int ROWB>
__global__ void __launch_bounds__(YOCOPP_COMPOSE_THREADS, YOCOPP_COMPOSE_CTAS_PER_SM) compose_append_kernel(ComposeParams p) {
    constexpr int CPR = ROWB / 16;                 // 16-byte chunks per (token, head) row
    constexpr int U = YOCOPP_COMPOSE_UNROLL;       // chunks in flight per thread
    extern __shared__ int s_cu[];   // staged prefix offsets (ragged batches only)

    if (p.cu_new != nullptr) {
        for (int i = threadIdx.x; i <= p.batch; i += blockDim.x) s_cu[i] = p.cu_new[i];
        __syncthreads();
    }
    const int64_t nchunks = p.total_rows * CPR;
    const ComposeCoef ck = make_coef(p.ak1, p.ak2, p.lam);
    const ComposeCoef cv = make_coef(p.av1, p.av2, p.lam);
    int bc = 0;  // ragged batches: this thread's last sequence (its chunks only move forward)
    // the sequence of token tok: the largest b with s_cu[b] <= tok (skips empty sequences), a few
    // steps on from this thread's last one, else a binary search
    auto seq_of = [&](int64_t tok) {
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
        return bc;
    };

    if (nchunks < (int64_t(1) << 31)) {
        // chunks, rows and tokens below 2^31: 32-bit indices, divisions by multiply-high; the cache
        // rows of an accepted cache are below 2^31 too
        const uint32_t n32 = uint32_t(nchunks), st32 = gridDim.x * blockDim.x;
        const uint32_t bs_mask = (1u << p.bs_log2) - 1u;
        for (uint32_t i0 = blockIdx.x * blockDim.x + threadIdx.x; i0 < n32; i0 += st32 * U) {
            uint4 x1k[U], xik[U], x1v[U], xiv[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const uint32_t idx = i0 + u * st32;
                if (idx < n32) {
                    const size_t off = size_t(idx) * 16;  // chunk idx of the packed [row][CPR] input
                    x1k[u] = ld_stream(p.k1 + off);
                    xik[u] = ld_stream(p.ki + off);
                    x1v[u] = ld_stream(p.v1 + off);
                    xiv[u] = ld_stream(p.vi + off);
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const uint32_t idx = i0 + u * st32;
                if (idx >= n32) continue;
                const uint32_t row = idx / CPR, c = idx % CPR;
                const uint32_t tok = fast_div(row, p.hkv_m, p.hkv_s);
                const uint32_t h = row - tok * uint32_t(p.hkv);
                uint32_t b, j;
                if (p.cu_new == nullptr) {
                    b = fast_div(tok, p.nu_m, p.nu_s);
                    j = tok - b * uint32_t(p.n_uniform);
                } else {
                    b = uint32_t(seq_of(tok));
                    j = tok - uint32_t(s_cu[b]);
                }
                const int position = __ldg(p.pos + b) + int(j);
                if (position < 0 || position >= p.capacity) {
                    record_status(YOCOPP_ECAPACITY);
                    continue;
                }
                uint32_t crow;
                if (p.block_table == nullptr) {
                    crow = (b * uint32_t(p.hkv) + h) * uint32_t(p.capacity) + uint32_t(position);
                } else {
                    const int blk = __ldg(p.block_table + size_t(b) * p.mbps + (uint32_t(position) >> p.bs_log2));
                    if (blk < 0 || blk >= p.num_blocks) {
                        record_status(YOCOPP_EDEVICE_CHECK);
                        continue;
                    }
                    crow = ((uint32_t(blk) * uint32_t(p.hkv) + h) << p.bs_log2) + (uint32_t(position) & bs_mask);
                }
                const size_t dst = size_t(crow) * ROWB + c * 16;
                st_global(p.ck + dst, compose_chunk<T>(x1k[u], xik[u], ck));
                st_global(p.cv + dst, compose_chunk<T>(x1v[u], xiv[u], cv));
            }
        }
        return;
    }

    const int64_t stride = int64_t(gridDim.x) * blockDim.x;
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
            const int64_t tok = row / p.hkv;
            const int h = int(row % p.hkv);
            int b, j;
            if (p.cu_new == nullptr) {
                b = int(tok / p.n_uniform);
                j = int(tok - int64_t(b) * p.n_uniform);
            } else {
                b = seq_of(tok);
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
