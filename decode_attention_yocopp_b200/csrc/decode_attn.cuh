// Split-K GQA decode attention over the shared cross-decoder cache
// (CUDA-core score product; decode_attn_tc.cuh moves the scores to tcgen05
// for bf16 / head_dim 128 and reuses this file's merge and helpers).
//
// You Only Cache Once (abstract): the cross-decoder reuses the self-decoder's
// cache through cross-attention.  YOCO++ section 2: every upper-half layer
// reads the middle layer's composed cache (K'_{L/2}, V'_{L/2}); section 3
// ("efficiency analysis"): decoding reads exactly one KV set per layer, so a
// decode step is bound by HBM bandwidth on these reads.
//
// Work decomposition.  The (sequence, kv-head) planes are cut into TILE-token
// tiles and flattened in (b, g, tile) order.  A persistent grid (a fixed number of CTAs
// per SM) takes equal contiguous ranges of that list, so any length mix is
// balanced to within one tile and each CTA streams contiguous K/V.  A CTA
// keeps online-softmax state for the (b, g) "segment" it is in; at the end of
// a segment it writes either the final output (segment = the whole plane) or
// an unnormalised partial (max, sum of exponentials, weighted value sum) to a
// workspace slot; the last CTA to finish a plane that spans several CTAs
// (counted with an atomic arrival counter) merges its partials with an exact
// log-sum-exp and writes the output.  One launch per layer.
//
// Inside a CTA.  One producer warp issues TMA tile loads (128-byte swizzled
// boxes, so the compute warps read shared memory without bank conflicts) into
// a STAGES-deep ring guarded by full/empty mbarriers.  W consumer warps split
// every tile's tokens.  Scores: 8 lanes per token, each lane holding 1/8 of
// the G query heads' channels in registers, packed fp32x2 FMAs, then a 3-step
// shuffle reduce-scatter that leaves every lane with one head's full score.
// Online softmax in the log2 domain (q is pre-scaled by scale * log2 e):
// warp-shuffle maxima, exp2, rescaling of the running sums.  Values: lanes
// own 16-byte channel chunks, probabilities broadcast from shared memory,
// packed FMAs into G x (channels per lane) fp32 accumulators.  All waits are
// bounded; on timeout the kernel records YOCOPP_ETIMEOUT and returns.
#pragma once

#include "common.cuh"

namespace yocopp {

struct DecodeParams {
    const uint8_t* q;
    uint8_t* out;
    const int32_t* seq_lens;
    const int32_t* block_table;  // nullptr: contiguous cache
    unsigned long long* ws_gen;  // workspace header: [0] generation of the last finished call, [1] call arrivals
    unsigned long long* ws_cnt;  // [batch * hkv] arrival counters: (call epoch << 20) | CTAs arrived
    float* ws_m;                 // [slots][G]
    float* ws_l;                 // [slots][G]
    float* ws_o;                 // [slots][G][D]
    float qscale;                // softmax scale * log2(e)
    int32_t batch, hkv, hq, capacity, block_size, mbps, num_blocks, boxr;
    int32_t num_ctas;
    int32_t seg_units;           // split plan: tiles' worth of work a segment's flush costs
    int32_t drop_tile;           // testing: a tile whose load is never issued (-1: none)
    int32_t prefetch;            // 0: skip the L2 prefetch of the first tiles (testing)
    uint64_t wait_limit_ns;
    float* part_out;             // non-null: write unnormalised [batch][hq][D + 2] (o, m, l) instead of out
    float fa1k, fa2k, fa1v, fa2v;  // read-time composition (fused variant): lambda * alpha
};

struct TileMeta {
    int32_t b, g, k, len, flags, pad;
};
enum : int32_t { kFirst = 1, kLast = 2, kWhole = 4 };

// FUSED: the stage also holds the layer-1 K/V tiles and K'/V' are composed at
// read time (twice the bytes per token, so the tile is halved).
template <int D, typename T, bool FUSED = false>
struct DecodeShape {
    static constexpr int EB = sizeof(T);
    static constexpr int ROWB = D * EB;                   // bytes per (token, head) row
    static constexpr int TILE = (ROWB <= 256 ? 64 : 32) / (FUSED ? 2 : 1);  // tokens per pipeline tile
    static constexpr int NBOX = ROWB / 128;               // 128-byte swizzle boxes per row
    static constexpr int BOXB = TILE * 128;               // bytes of one box column of a tile
    static constexpr int KV_BYTES = TILE * ROWB;          // one K (or V) tile
    static constexpr int NSRC = FUSED ? 4 : 2;            // tiles per stage: K, V (, K_1, V_1)
    static constexpr int STAGE_BYTES = NSRC * KV_BYTES;
    static constexpr int CPR = ROWB / 16;                 // 16-byte chunks per row
    static constexpr int CPL = CPR / 8;                   // score phase: chunks per lane
    static constexpr int EPC = 16 / EB;                   // elements per chunk
    static constexpr int TPI = 32 / CPR;                  // value phase: tokens per warp step
};

constexpr float NEG_INF_F = -INFINITY;

// Final result of one (sequence, query head, channel): the normalised output,
// or (partial mode) the unnormalised weighted sum plus, at channel 0, the
// head's maximum (log2 units) and sum of exponentials.
template <typename T, int D>
__device__ __forceinline__ void emit(const DecodeParams& p, int64_t row, int c, float M, float Ls, float O) {
    if (p.part_out != nullptr) {
        float* r = p.part_out + row * (D + 2);
        r[c] = O;
        if (c == 0) {
            r[D] = M;
            r[D + 1] = Ls;
        }
        return;
    }
    const float y = Ls > 0.f ? O / Ls : 0.f;
    if constexpr (sizeof(T) == 2)
        reinterpret_cast<__nv_bfloat16*>(p.out)[row * D + c] = __float2bfloat16_rn(y);
    else
        reinterpret_cast<float*>(p.out)[row * D + c] = y;
}

template <typename T>
__device__ __forceinline__ void write_out(uint8_t* out, int64_t i, float y) {
    if constexpr (sizeof(T) == 2)
        reinterpret_cast<__nv_bfloat16*>(out)[i] = __float2bfloat16_rn(y);
    else
        reinterpret_cast<float*>(out)[i] = y;
}

__device__ __forceinline__ int ntiles_of(int len, int tile) { return (len + tile - 1) / tile; }

__device__ __forceinline__ int clamp_len(const int32_t* lens, int b, int cap) {
    int len = __ldg(lens + b);
    return len < 0 ? 0 : (len > cap ? cap : len);
}

// Rendezvous of the first nthr threads of the block (nthr a multiple of 32).
__device__ __forceinline__ void sync_first(int nthr) { asm volatile("bar.sync 1, %0;" ::"r"(nthr) : "memory"); }

// Exclusive prefix of tiles per sequence (x kv heads) into s_ts[0..batch], by the
// block's first nthr threads.
template <int TILE>
__device__ void tile_prefix(const DecodeParams& p, int* s_ts, int* s_warp, int nthr) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int per = (p.batch + nthr - 1) / nthr;
    const int b0 = min(tid * per, p.batch), b1 = min(b0 + per, p.batch);
    int sum = 0;
    for (int b = b0; b < b1; ++b) {
        const int raw = __ldg(p.seq_lens + b);
        if (blockIdx.x == 0 && (raw < 0 || raw > p.capacity)) record_status(YOCOPP_ECAPACITY);
        sum += ntiles_of(clamp_len(p.seq_lens, b, p.capacity), TILE) * p.hkv;
    }
    int x = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) s_warp[warp] = x;
    sync_first(nthr);
    if (warp == 0) {
        int v = lane < (nthr >> 5) ? s_warp[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, v, o);
            if (lane >= o) v += y;
        }
        s_warp[lane] = v;
    }
    sync_first(nthr);
    int excl = x - sum + (warp > 0 ? s_warp[warp - 1] : 0);
    for (int b = b0; b < b1; ++b) {
        s_ts[b] = excl;
        excl += ntiles_of(clamp_len(p.seq_lens, b, p.capacity), TILE) * p.hkv;
    }
    if (tid == nthr - 1) s_ts[p.batch] = excl;
    sync_first(nthr);
}

// Split plan.  The tiles of all (sequence, kv-head) planes are flattened in
// (b, g, tile) order, and plane P = b * hkv + g is preceded by `seg` extra
// units: what closing a segment (flushing a partial, arriving, perhaps
// merging) costs a CTA, in tiles.  CTA c takes the tiles whose units fall in
// [c * unit, (c + 1) * unit), unit = ceil((tiles + seg * planes) / CTAs), so a
// CTA that closes more segments streams fewer tiles and the CTAs finish
// together.  unit_of(t) = t + seg * (P(t) + 1) is increasing in t.
struct SplitPlan {
    int total;  // tiles
    int unit;   // units per CTA (>= 1)
    int seg;    // units per plane start
};

__device__ __forceinline__ SplitPlan make_plan(const DecodeParams& p, const int* s_ts, int seg) {
    SplitPlan sp;
    sp.total = s_ts[p.batch];
    sp.seg = seg;
    const int64_t units = int64_t(sp.total) + int64_t(seg) * p.batch * p.hkv;
    sp.unit = int((units + p.num_ctas - 1) / p.num_ctas);
    if (sp.unit < 1) sp.unit = 1;
    return sp;
}

// The first tile whose unit is >= u (sp.total if none): binary search for the
// last plane starting at or before u, then the offset inside it.
__device__ __forceinline__ int plan_tile_at(const DecodeParams& p, const int* s_ts, const SplitPlan& sp, int64_t u) {
    const int planes = p.batch * p.hkv;
    if (u >= int64_t(sp.total) + int64_t(sp.seg) * planes) return sp.total;
    auto first_tile = [&](int P) {  // first tile of plane P
        const int b = P / p.hkv, g = P - b * p.hkv;
        return s_ts[b] + g * ((s_ts[b + 1] - s_ts[b]) / p.hkv);
    };
    int lo = 0, hi = planes;  // start unit of plane lo <= u < start unit of plane hi
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (int64_t(first_tile(mid)) + int64_t(sp.seg) * mid <= u) lo = mid; else hi = mid;
    }
    const int f = first_tile(lo);
    const int64_t into = u - (int64_t(f) + int64_t(sp.seg) * (lo + 1));  // units past its cost units
    const int t = into > 0 ? int(f + into) : f;
    return min(t, sp.total);
}

// The CTA whose range holds tile t of plane P.
__device__ __forceinline__ int plan_cta_of(const SplitPlan& sp, int t, int P) {
    return int((int64_t(t) + int64_t(sp.seg) * (P + 1)) / sp.unit);
}

// This CTA's tile range [start, end): lanes 0 and 1 search, the warp shares.
__device__ __forceinline__ int2 plan_range(const DecodeParams& p, const int* s_ts, const SplitPlan& sp, int lane) {
    int v = 0;
    if (lane < 2) v = plan_tile_at(p, s_ts, sp, int64_t(blockIdx.x + lane) * sp.unit);
    return make_int2(__shfl_sync(0xffffffffu, v, 0), __shfl_sync(0xffffffffu, v, 1));
}

// ---- the first tiles, prefetched before the previous kernel has finished ---
// A kernel launched as a programmatic dependent may start while the previous
// kernel still runs, and may read its inputs only after griddep_wait.  Until
// then one warp guesses this CTA's plan from the lengths and block tables as
// they stand (gpu-scope relaxed loads, which may be stale) and prefetches the
// first tiles of its range into L2, so that the kernel's HBM reads start in
// the previous kernel's tail.  The guess steers prefetches only: a stale length
// or block costs a useless prefetch, never a wrong result, since everything the
// kernel computes reads the inputs again after the wait.
constexpr int kGuessMaxBatch = 256;  // larger batches skip the prefetch

// The warp's guess of the prefix of tiles into s_g[0..batch], then L2 prefetches of
// the first npf (<= 32) tiles of the guessed range.
template <int TILE, int NBOX, int NSB_MAX>
__device__ void prefetch_first_tiles(const DecodeParams& p, const CUtensorMap* tmK, const CUtensorMap* tmV,
                                     int* s_g, int npf, int lane) {
    constexpr int PER = kGuessMaxBatch / 32;
    int n[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        const int b = i * 32 + lane;
        const int raw = b < p.batch ? ld_relaxed_gpu(p.seq_lens + b) : 0;
        n[i] = ntiles_of(raw < 0 ? 0 : min(raw, p.capacity), TILE) * p.hkv;
    }
    int base = 0;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        if (i * 32 >= p.batch) break;
        int x = n[i];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (i * 32 + lane < p.batch) s_g[i * 32 + lane] = base + x - n[i];
        base += __shfl_sync(0xffffffffu, x, 31);
    }
    if (lane == 0) s_g[p.batch] = base;
    __syncwarp();
    const SplitPlan sp = make_plan(p, s_g, p.seg_units);
    const int2 range = plan_range(p, s_g, sp, lane);
    const int t = range.x + lane;
    if (lane >= npf || t >= range.y) return;
    int lo = 0, hi = p.batch;  // s_g[lo] <= t < s_g[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (s_g[mid] <= t) lo = mid; else hi = mid;
    }
    const int b = lo;
    const int nt = (s_g[b + 1] - s_g[b]) / p.hkv;  // > 0: tile t lies in sequence b
    const int local = t - s_g[b];
    const int g = local / nt, k = local - g * nt;
    if (p.block_table == nullptr) {
        const int row = (b * p.hkv + g) * p.capacity + k * TILE;
#pragma unroll
        for (int bx = 0; bx < NBOX; ++bx) {
            tma_prefetch_2d(tmK, bx * 64, row);
            tma_prefetch_2d(tmV, bx * 64, row);
        }
        return;
    }
    const int raw = ld_relaxed_gpu(p.seq_lens + b);
    const int len = raw < 0 ? 0 : min(raw, p.capacity);
    const int nsb = TILE / p.boxr;
#pragma unroll
    for (int s = 0; s < NSB_MAX; ++s) {
        const int tok = k * TILE + s * p.boxr;
        if (s >= nsb || tok >= len) continue;
        const int blk = ld_relaxed_gpu(p.block_table + int64_t(b) * p.mbps + tok / p.block_size);
        if (blk < 0 || blk >= p.num_blocks) continue;
        const int row = (blk * p.hkv + g) * p.block_size + tok % p.block_size;
#pragma unroll
        for (int bx = 0; bx < NBOX; ++bx) {
            tma_prefetch_2d(tmK, bx * 64, row);
            tma_prefetch_2d(tmV, bx * 64, row);
        }
    }
}

template <typename T, int D, int G, int W, int STAGES, bool FUSED = false>
struct DecodeSmem {
    using S = DecodeShape<D, T, FUSED>;
    static constexpr int TPW = S::TILE / W;
    static constexpr size_t up16(size_t x) { return (x + 15) & ~size_t(15); }
    static constexpr size_t kStages = size_t(STAGES) * S::STAGE_BYTES;      // 1024-aligned ring
    static constexpr size_t kBars = kStages;                                 // full[S], empty[S], sync
    static constexpr size_t kMeta = up16(kBars + (2 * STAGES + 2) * sizeof(uint64_t));  // + sync, merge
    static constexpr size_t kP = up16(kMeta + STAGES * sizeof(TileMeta));
    static constexpr size_t kMergeM = up16(kP + size_t(W) * TPW * G * sizeof(float2));
    static constexpr size_t kMergeL = up16(kMergeM + size_t(W) * G * sizeof(float));
    static constexpr size_t kMergeO = up16(kMergeL + size_t(W) * G * sizeof(float));
    static constexpr size_t kTileStart = up16(kMergeO + size_t(W) * G * D * sizeof(float));
    static size_t bytes(int batch) { return 1024 + kTileStart + size_t(batch + 1) * sizeof(int); }
};

// This call's epoch, read from the workspace header by each CTA at start.
// header[0] = the epoch of the last call that every CTA joined (0 in a
// zero-filled workspace); header[1] = (epoch << 20) | CTAs of the current call
// that have read it.  Each CTA reads header[0], takes epoch = header[0] + 1,
// and arrives on header[1]; the last CTA to arrive publishes the epoch in
// header[0] for the next call.  Every CTA arrives right after reading, before
// any work that could time out, so each call advances the epoch exactly once;
// the epoch lives on the device, so a captured CUDA graph replays correctly.
// The arrival half of join_call, for a CTA that read the epoch (header[0] + 1)
// earlier: any time after that read will do.
__device__ __forceinline__ void arrive_call(unsigned long long* hdr, unsigned long long epoch, unsigned num_ctas) {
    __threadfence();
    atomicMax(hdr + 1, epoch << 20);
    const unsigned long long old = atomicAdd(hdr + 1, 1ull);
    if ((old >> 20) == epoch && unsigned(old & 0xFFFFFull) + 1u == num_ctas) {
        __threadfence();
        atomicMax(hdr, epoch);
    }
}

__device__ __forceinline__ unsigned long long join_call(unsigned long long* hdr, unsigned num_ctas) {
    const unsigned long long epoch = __ldcg(hdr) + 1ull;
    arrive_call(hdr, epoch, num_ctas);
    return epoch;
}

// Arrive on a plane's counter for this call; returns how many CTAs have arrived
// (this one included), or 0 if the counter holds a later call's tag (a
// workspace that was not zero-filled before its first use).  The word is
// (epoch << 20) | count.  Epochs only grow, so atomicMax replaces a tag left by
// any earlier call (finished or aborted) with this call's tag and a zero
// count; two single atomics, no retry loop.
__device__ __forceinline__ unsigned arrive_plane(unsigned long long* cnt, unsigned long long epoch) {
    atomicMax(cnt, epoch << 20);
    const unsigned long long old = atomicAdd(cnt, 1ull);
    if ((old >> 20) != epoch) return 0;
    return unsigned(old & 0xFFFFFull) + 1u;
}

// Per-warp state and work of a consumer warp: the group's queries in
// registers, the online-softmax running maxima / partial sums, and the
// running weighted value sums for this warp's share of every tile.
// One 16-byte chunk of a K or V tile as EPC/2 fp32 pairs; with FUSED, composed
// at read time from the layer-L/2 and layer-1 tiles: (lambda a2) xi + (lambda a1) x1.
template <typename T, bool FUSED, int NP>
__device__ __forceinline__ void load_pairs(const uint8_t* a, const uint8_t* a1, float2 c1, float2 c2,
                                           float2 (&out)[NP]) {
    const uint4 v = *reinterpret_cast<const uint4*>(a);
    const uint32_t* w = reinterpret_cast<const uint32_t*>(&v);
    if constexpr (sizeof(T) == 2) {
#pragma unroll
        for (int e = 0; e < 4; ++e) out[e] = bf16x2_to_float2(w[e]);
    } else {
        out[0] = make_float2(__uint_as_float(w[0]), __uint_as_float(w[1]));
        out[1] = make_float2(__uint_as_float(w[2]), __uint_as_float(w[3]));
    }
    if constexpr (FUSED) {
        const uint4 v1 = *reinterpret_cast<const uint4*>(a1);
        const uint32_t* w1 = reinterpret_cast<const uint32_t*>(&v1);
#pragma unroll
        for (int e = 0; e < NP; ++e) {
            float2 x1;
            if constexpr (sizeof(T) == 2)
                x1 = bf16x2_to_float2(w1[e]);
            else
                x1 = make_float2(__uint_as_float(w1[2 * e]), __uint_as_float(w1[2 * e + 1]));
            out[e] = ffma2(c1, x1, fmul2(c2, out[e]));
        }
    }
}

template <typename T, int D, int G, int W, bool FUSED = false>
struct ConsumerWarp {
    using S = DecodeShape<D, T, FUSED>;
    static constexpr int TILE = S::TILE, TPW = TILE / W, CPR = S::CPR, CPL = S::CPL, EPC = S::EPC, TPI = S::TPI;
    static constexpr int QK_IT = TPW / 4;     // score steps (4 tokens per step)
    static constexpr int PV_IT = TPW / TPI;   // value steps (TPI tokens per step)
    static constexpr int HL = 8 / G;          // lanes holding one head's score after the reduce-scatter
    static_assert(G == 1 || G == 2 || G == 4, "group size");
    static_assert(TPW % 4 == 0 && TPW % TPI == 0, "tile split");

    float2 q2[G][CPL * EPC / 2];  // q * scale * log2(e), this lane's channels
    float2 acc[G][EPC / 2];       // running sum of p * v, this lane's channel chunk
    float m_run[G];               // running maximum per head (warp-uniform)
    float l_part;                 // running sum of p for head hr over this lane's tokens
    float m_mine;                 // m_run[hr], kept as a scalar (an indexed read would spill the state)
    const int warp, lane, j4, r8, hr, pc, pslot, pbx, pcc;

    __device__ __forceinline__ ConsumerWarp(int warp_, int lane_)
        : warp(warp_), lane(lane_), j4(lane_ >> 3), r8(lane_ & 7), hr((lane_ & 7) / HL), pc(lane_ % CPR),
          pslot(lane_ / CPR), pbx((lane_ % CPR) >> 3), pcc((lane_ % CPR) & 7) {}

    // New (sequence, kv-head) segment: reset the state and load the group's queries.
    __device__ __forceinline__ void begin_segment(const DecodeParams& p, int b, int g) {
#pragma unroll
        for (int h = 0; h < G; ++h) {
            m_run[h] = NEG_INF_F;
#pragma unroll
            for (int e = 0; e < EPC / 2; ++e) acc[h][e] = make_float2(0.f, 0.f);
            const uint8_t* qrow = p.q + (int64_t(b) * p.hq + g * G + h) * S::ROWB;
#pragma unroll
            for (int jb = 0; jb < CPL; ++jb) {
                const uint4 v = ld_stream(qrow + (r8 + 8 * jb) * 16);
                const uint32_t* w = reinterpret_cast<const uint32_t*>(&v);
                if constexpr (S::EB == 2) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 f = bf16x2_to_float2(w[e]);
                        q2[h][jb * 4 + e] = make_float2(f.x * p.qscale, f.y * p.qscale);
                    }
                } else {
                    q2[h][jb * 2 + 0] = make_float2(__uint_as_float(w[0]) * p.qscale, __uint_as_float(w[1]) * p.qscale);
                    q2[h][jb * 2 + 1] = make_float2(__uint_as_float(w[2]) * p.qscale, __uint_as_float(w[3]) * p.qscale);
                }
            }
        }
        l_part = 0.f;
        m_mine = NEG_INF_F;
    }

    float2 fk1, fk2, fv1, fv2;    // read-time composition coefficients (fused variant)

    // Score of one token row for head hr (8 lanes per token, packed FMAs, reduce-scatter).
    __device__ __forceinline__ float score(const uint8_t* Kt, const uint8_t* K1t, int row) const {
        float2 part[G];
#pragma unroll
        for (int h = 0; h < G; ++h) part[h] = make_float2(0.f, 0.f);
#pragma unroll
        for (int jb = 0; jb < CPL; ++jb) {
            const int off = jb * S::BOXB + row * 128 + ((r8 ^ (row & 7)) << 4);
            float2 kf[EPC / 2];
            load_pairs<T, FUSED>(Kt + off, K1t + off, fk1, fk2, kf);
#pragma unroll
            for (int e = 0; e < EPC / 2; ++e)
#pragma unroll
                for (int h = 0; h < G; ++h) part[h] = ffma2(q2[h][jb * (EPC / 2) + e], kf[e], part[h]);
        }
        float v[G];
#pragma unroll
        for (int h = 0; h < G; ++h) v[h] = part[h].x + part[h].y;
        float sc;
        if constexpr (G == 4) {
            const bool up = r8 & 4;
            float k0 = up ? v[2] : v[0], k1 = up ? v[3] : v[1];
            const float s0 = up ? v[0] : v[2], s1 = up ? v[1] : v[3];
            k0 += __shfl_xor_sync(0xffffffffu, s0, 4);
            k1 += __shfl_xor_sync(0xffffffffu, s1, 4);
            const bool up2 = r8 & 2;
            sc = up2 ? k1 : k0;
            sc += __shfl_xor_sync(0xffffffffu, up2 ? k0 : k1, 2);
            sc += __shfl_xor_sync(0xffffffffu, sc, 1);
        } else if constexpr (G == 2) {
            const bool up = r8 & 4;
            sc = up ? v[1] : v[0];
            sc += __shfl_xor_sync(0xffffffffu, up ? v[0] : v[1], 4);
            sc += __shfl_xor_sync(0xffffffffu, sc, 2);
            sc += __shfl_xor_sync(0xffffffffu, sc, 1);
        } else {
            sc = v[0];
            sc += __shfl_xor_sync(0xffffffffu, sc, 4);
            sc += __shfl_xor_sync(0xffffffffu, sc, 2);
            sc += __shfl_xor_sync(0xffffffffu, sc, 1);
        }
        return sc;
    }

    // One tile: scores, online-softmax update, values.  MASK: the slice holds
    // tokens at or past len (the last tile of a sequence).
    template <bool MASK>
    __device__ __forceinline__ void tile(const uint8_t* Kt, const uint8_t* Vt, float2* p2, int tok0, int len) {
        const int rbase = warp * TPW;
        const uint8_t* K1t = Kt + 2 * S::KV_BYTES;  // layer-1 tiles (fused variant only)
        const uint8_t* V1t = Kt + 3 * S::KV_BYTES;
        float s[QK_IT];
#pragma unroll
        for (int i = 0; i < QK_IT; ++i) {
            s[i] = score(Kt, K1t, rbase + i * 4 + j4);
            if (MASK && tok0 + i * 4 + j4 >= len) s[i] = NEG_INF_F;
        }
        // maxima of this slice per head, then the (warp-uniform) running update
        float mloc = s[0];
#pragma unroll
        for (int i = 1; i < QK_IT; ++i) mloc = fmaxf(mloc, s[i]);
        mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, 8));
        mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, 16));
        float mnew[G];
        bool grow = false;
#pragma unroll
        for (int h = 0; h < G; ++h) {
            mnew[h] = fmaxf(m_run[h], __shfl_sync(0xffffffffu, mloc, h * HL));
            grow |= mnew[h] > m_run[h];
        }
        if (grow) {  // rescale only when some maximum rose
#pragma unroll
            for (int h = 0; h < G; ++h) {
                const float corr = mnew[h] == NEG_INF_F ? 1.f : exp2f(m_run[h] - mnew[h]);
                m_run[h] = mnew[h];
                const float2 c2 = make_float2(corr, corr);
#pragma unroll
                for (int e = 0; e < EPC / 2; ++e) acc[h][e] = fmul2(acc[h][e], c2);
                if (h == hr) {
                    l_part *= corr;
                    m_mine = mnew[h];
                }
            }
        }
#pragma unroll
        for (int i = 0; i < QK_IT; ++i) {
            const float pr = (MASK && s[i] == NEG_INF_F) ? 0.f : exp2f(s[i] - m_mine);
            l_part += pr;
            if (r8 % HL == 0) p2[(i * 4 + j4) * G + hr] = make_float2(pr, pr);
        }
        __syncwarp();

        // values: acc[h] += p[h] * v over the slice (TPI tokens per step)
#pragma unroll
        for (int i2 = 0; i2 < PV_IT; ++i2) {
            const int tl = i2 * TPI + pslot;  // token within the slice
            const int tk = rbase + tl;        // row within the tile
            const int voff = pbx * S::BOXB + tk * 128 + ((pcc ^ (tk & 7)) << 4);
            float2 vf[EPC / 2];
            load_pairs<T, FUSED>(Vt + voff, V1t + voff, fv1, fv2, vf);
            if (MASK && tok0 + tl >= len) {  // never use rows past the sequence
#pragma unroll
                for (int e = 0; e < EPC / 2; ++e) vf[e] = make_float2(0.f, 0.f);
            }
            float2 pp[G];
            if constexpr (G >= 2) {
#pragma unroll
                for (int h = 0; h < G; h += 2) {
                    const float4 t4 = *reinterpret_cast<const float4*>(p2 + tl * G + h);
                    pp[h] = make_float2(t4.x, t4.y);
                    pp[h + 1] = make_float2(t4.z, t4.w);
                }
            } else {
                pp[0] = p2[tl];
            }
#pragma unroll
            for (int h = 0; h < G; ++h)
#pragma unroll
                for (int e = 0; e < EPC / 2; ++e) acc[h][e] = ffma2(pp[h], vf[e], acc[h][e]);
        }
        __syncwarp();  // p2 is rewritten by the next tile
    }

    // Reduce this warp's state over its lanes and store it for the CTA merge.
    __device__ __forceinline__ void stash(float* mg_m, float* mg_l, float* mg_o) {
        float lsum = (r8 % HL == 0) ? l_part : 0.f;
        lsum += __shfl_xor_sync(0xffffffffu, lsum, 8);
        lsum += __shfl_xor_sync(0xffffffffu, lsum, 16);
#pragma unroll
        for (int o = CPR; o < 32; o <<= 1)
#pragma unroll
            for (int h = 0; h < G; ++h)
#pragma unroll
                for (int e = 0; e < EPC / 2; ++e) {
                    acc[h][e].x += __shfl_xor_sync(0xffffffffu, acc[h][e].x, o);
                    acc[h][e].y += __shfl_xor_sync(0xffffffffu, acc[h][e].y, o);
                }
#pragma unroll
        for (int h = 0; h < G; ++h) {
            const float lh = __shfl_sync(0xffffffffu, lsum, h * HL);
            if (lane == 0) {
                mg_m[warp * G + h] = m_run[h];
                mg_l[warp * G + h] = lh;
            }
            if (lane < CPR) {
#pragma unroll
                for (int e = 0; e < EPC / 2; ++e)
                    *reinterpret_cast<float2*>(mg_o + (warp * G + h) * D + lane * EPC + 2 * e) = acc[h][e];
            }
        }
    }
};

// Shared memory the last CTA of a plane may stage that plane's partial value
// sums in (the tile ring, free once the CTA has consumed its last tile), with
// an mbarrier for the bulk copy; buf == nullptr: no staging.
struct MergeStage {
    uint8_t* buf;
    uint32_t bytes;
    uint64_t* bar;
};

// Merge the partials of one (sequence, kv-head) plane written by CTAs c0..c1
// (slots plane + cta) and write the group's outputs.  Run by the W consumer
// warps of the last CTA to arrive.  One parallel pass stages every part's
// maximum and sum in shared memory (the probability and warp-merge areas,
// free at this point); after one rendezvous, the lanes that hold a head's
// channels form its maximum, the weights 2^(m_s - M) (once per part and head)
// and the normaliser among themselves, and each thread accumulates its 4
// channels.  With a staging area large enough,
// the parts' value sums (contiguous slots) come in with one bulk copy issued
// first, so that the whole merge costs one round trip to L2 for them instead
// of one per few parts.
// own >= 0: part `own` (this CTA's) was not published; its state is the W
// consumer warps' stash (mg_m, mg_l: [W][G], mg_o: [W][G][D]) and is merged
// from there.
template <int D, int G, int W>
__device__ __forceinline__ void own_state(const float* mg_m, const float* mg_l, int h, float& M, float& Ls) {
    M = NEG_INF_F;
#pragma unroll
    for (int w2 = 0; w2 < W; ++w2) M = fmaxf(M, mg_m[w2 * G + h]);
    Ls = 0.f;
    if (M != NEG_INF_F) {
#pragma unroll
        for (int w2 = 0; w2 < W; ++w2) Ls += exp2f(mg_m[w2 * G + h] - M) * mg_l[w2 * G + h];
    }
}

template <typename T, int D, int G, int W, typename Sync>
__device__ __forceinline__ bool merge_plane(const DecodeParams& p, int bg, int c0, int c1, int64_t out_row0,
                                            float* scratch, int scratch_floats, Sync& sync, int tid,
                                            const MergeStage* stage, int own = -1, const float* mg_m = nullptr,
                                            const float* mg_l = nullptr, const float* mg_o = nullptr) {
    constexpr int NT = W * 32;
    const int nparts = c1 - c0 + 1;
    const int cap = scratch_floats / (2 * G);  // parts whose maxima and sums fit the scratch
    const float* pm = p.ws_m + int64_t(bg + c0) * G;
    const float* pl = p.ws_l + int64_t(bg + c0) * G;
    const float4* po = reinterpret_cast<const float4*>(p.ws_o + int64_t(bg + c0) * G * D);
    if (nparts > cap && own < 0) {
        // very many splits of one plane: per-element loop without staging
        for (int idx = tid; idx < G * D; idx += NT) {
            const int h = idx / D, c = idx % D;
            float M = NEG_INF_F;
            for (int s2 = 0; s2 < nparts; ++s2) M = fmaxf(M, __ldcg(pm + s2 * G + h));
            float Ls = 0.f, O = 0.f;
            for (int s2 = 0; s2 < nparts; ++s2) {
                const float f = exp2f(__ldcg(pm + s2 * G + h) - M);
                Ls += f * __ldcg(pl + s2 * G + h);
                O += f * __ldcg(p.ws_o + (int64_t(bg + c0 + s2) * G + h) * D + c);
            }
            emit<T, D>(p, out_row0 + h, c, M, Ls, O);
        }
        return true;
    }
    const uint32_t obytes = uint32_t(nparts) * G * D * 4;
    const bool staged = stage != nullptr && stage->buf != nullptr && obytes <= stage->bytes;
    if (staged && tid == 0) {
        fence_proxy_async_global();  // the parts were written (and acquired) through the generic proxy
        mbar_arrive_expect_tx(stage->bar, obytes);
        bulk_load(stage->buf, po, obytes, stage->bar);
    }
    float* wts = scratch;                   // [part][G]: maxima, then weights
    float* lss = scratch + cap * G;         // [part][G]: sums of exponentials
    for (int i = tid; i < nparts * G; i += NT) {
        if (i / G == own) {
            own_state<D, G, W>(mg_m, mg_l, i % G, wts[i], lss[i]);
        } else {
            wts[i] = __ldcg(pm + i);
            lss[i] = __ldcg(pl + i);
        }
    }
    bool ok = sync();
    if (staged) {
        // every thread waits (bounded) for the bulk copy; a warp continues only if all its lanes saw it
        ok = __all_sync(0xffffffffu, mbar_wait(stage->bar, 0, p.wait_limit_ns)) && ok;
        if (!ok) return false;
        po = reinterpret_cast<const float4*>(stage->buf);
    }
    // A thread holds 4 channels, so a head's D channels are LPH = D / 4 lanes of one warp; those
    // lanes form the head's maximum, weights 2^(m_s - M) (in place of the maxima, read back by
    // the same lanes) and normaliser among themselves, with shuffles and no rendezvous.
    constexpr int LPH = D / 4;
    static_assert(32 % LPH == 0, "a head's lanes within one warp");
    const int lane = tid & 31, g = lane % LPH;
    for (int q0 = tid - lane; q0 < G * D / 4; q0 += NT) {  // warp-uniform trip count
        const int q4 = q0 + lane;
        const bool act = q4 < G * D / 4;
        const int h = act ? (q4 * 4) / D : 0;
        float M = NEG_INF_F;
        if (act)
            for (int s2 = g; s2 < nparts; s2 += LPH) M = fmaxf(M, wts[s2 * G + h]);
#pragma unroll
        for (int o = LPH / 2; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o, LPH));
        float Ls = 0.f;
        if (act)
            for (int s2 = g; s2 < nparts; s2 += LPH) {
                const float f = M != NEG_INF_F ? exp2f(wts[s2 * G + h] - M) : 0.f;
                wts[s2 * G + h] = f;
                Ls += f * lss[s2 * G + h];
            }
#pragma unroll
        for (int o = LPH / 2; o > 0; o >>= 1) Ls += __shfl_xor_sync(0xffffffffu, Ls, o, LPH);
        __syncwarp();
        if (!act) continue;
        float4 O = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
        for (int s2 = 0; s2 < nparts; ++s2) {
            if (s2 == own) continue;
            const float4 o = staged ? po[int64_t(s2) * (G * D / 4) + q4] : __ldcg(po + int64_t(s2) * (G * D / 4) + q4);
            const float f = wts[s2 * G + h];
            O.x += f * o.x; O.y += f * o.y; O.z += f * o.z; O.w += f * o.w;
        }
        if (own >= 0) {
            // this CTA's part from the warps' stash, relative to its own maximum
            float Mo, Lo;
            own_state<D, G, W>(mg_m, mg_l, h, Mo, Lo);
            if (Mo != NEG_INF_F) {
                const float f = wts[own * G + h];
                const int c = (q4 * 4) % D;
#pragma unroll
                for (int w2 = 0; w2 < W; ++w2) {
                    const float fw = f * exp2f(mg_m[w2 * G + h] - Mo);
                    const float4 o = *reinterpret_cast<const float4*>(mg_o + (w2 * G + h) * D + c);
                    O.x += fw * o.x; O.y += fw * o.y; O.z += fw * o.z; O.w += fw * o.w;
                }
            }
        }
        const int c = (q4 * 4) % D;
        if (p.part_out != nullptr) {
            emit<T, D>(p, out_row0 + h, c + 0, M, Ls, O.x);
            emit<T, D>(p, out_row0 + h, c + 1, M, Ls, O.y);
            emit<T, D>(p, out_row0 + h, c + 2, M, Ls, O.z);
            emit<T, D>(p, out_row0 + h, c + 3, M, Ls, O.w);
        } else {
            const float inv = Ls > 0.f ? 1.f / Ls : 0.f;
            const int64_t o0 = out_row0 * D + int64_t(q4) * 4;
            write_out<T>(p.out, o0 + 0, O.x * inv);
            write_out<T>(p.out, o0 + 1, O.y * inv);
            write_out<T>(p.out, o0 + 2, O.z * inv);
            write_out<T>(p.out, o0 + 3, O.w * inv);
        }
    }
    return ok;
}

// End of a (sequence, kv-head) segment, after the warps' states are stashed in
// mg_*: merge them; write the output (whole plane) or this CTA's partial, then
// arrive on the plane's counter and, as the last CTA, merge the plane.  Run by
// the W consumer warps (ctid = consumer thread index).  False on a timed-out
// rendezvous.
template <typename T, int D, int G, int W, typename Sync>
__device__ __forceinline__ bool flush_segment(const DecodeParams& p, const TileMeta& mt, int ctid, const SplitPlan& sp,
                                              const int* s_ts, float* mg_m, float* mg_l, float* mg_o, float* scratch,
                                              int scratch_floats, Sync& consumer_sync, int& s_last,
                                              unsigned long long epoch, const MergeStage* stage = nullptr,
                                              int own_floats = 0, int snap_plane = -1,
                                              unsigned long long snap = 0) {
    if (!consumer_sync()) return false;
    const int bg = mt.b * p.hkv + mt.g;
    const int slot = bg + int(blockIdx.x);
    const bool whole = mt.flags & kWhole;
    // the fast merge below stages in the first own_floats of the scratch only (the rest holds
    // the warps' stash, which it still reads)
    const int own_cap = (own_floats - 2 * G) / (2 * G);
    if (!whole && stage != nullptr && own_cap > 0) {
        // The CTA's final segment: if every other part of the plane had arrived when ctid 0
        // read the plane's counter a few tiles ago (snap, snap_plane: held by ctid 0 only, so
        // every other condition here is uniform across the consumer threads), this CTA is the
        // last one and merges straight from its warps' stash, without publishing its part (no
        // fence and no arrival before the merge).
        const int nt = ntiles_of(mt.len, mt.pad);
        const int first = s_ts[mt.b] + mt.g * nt;
        const int c0 = plan_cta_of(sp, first, bg), c1 = plan_cta_of(sp, first + nt - 1, bg);
        if (c1 - c0 + 1 > own_cap) goto publish;
        if (ctid == 0) {
            const bool all_in = snap_plane == bg && (snap >> 20) == epoch &&
                                unsigned(snap & 0xFFFFFull) + 1u == unsigned(c1 - c0 + 1);
            if (all_in) fence_acq_rel_gpu();  // acquire what the relaxed read saw
            s_last = all_in ? 2 : 0;
        }
        if (!consumer_sync()) return false;
        if (s_last == 2) {
            if (!merge_plane<T, D, G, W>(p, bg, c0, c1, int64_t(mt.b) * p.hq + mt.g * G, scratch, own_floats,
                                         consumer_sync, ctid, stage, int(blockIdx.x) - c0, mg_m, mg_l, mg_o))
                return false;
            return consumer_sync();
        }
    }
publish:
    for (int idx = ctid; idx < G * D; idx += W * 32) {
        const int h = idx / D, c = idx % D;
        float M = NEG_INF_F;
#pragma unroll
        for (int w2 = 0; w2 < W; ++w2) M = fmaxf(M, mg_m[w2 * G + h]);
        float Ls = 0.f, O = 0.f;
        if (M != NEG_INF_F) {
#pragma unroll
            for (int w2 = 0; w2 < W; ++w2) {
                const float f = exp2f(mg_m[w2 * G + h] - M);
                Ls += f * mg_l[w2 * G + h];
                O += f * mg_o[(w2 * G + h) * D + c];
            }
        }
        if (whole) {
            emit<T, D>(p, int64_t(mt.b) * p.hq + mt.g * G + h, c, M, Ls, O);
        } else {
            p.ws_o[(int64_t(slot) * G + h) * D + c] = O;
            if (c == 0) {
                p.ws_m[int64_t(slot) * G + h] = M;
                p.ws_l[int64_t(slot) * G + h] = Ls;
            }
        }
    }
    if (!whole) {
        // publish this CTA's partial, count arrivals; the last CTA merges the plane
        __threadfence();
        if (!consumer_sync()) return false;
        const int nt = ntiles_of(mt.len, mt.pad);  // pad carries the kernel's tile size
        const int first = s_ts[mt.b] + mt.g * nt;
        const int c0 = plan_cta_of(sp, first, bg), c1 = plan_cta_of(sp, first + nt - 1, bg);
        if (ctid == 0) {
            const unsigned arrived = arrive_plane(p.ws_cnt + bg, epoch);
            if (arrived == 0) record_status(YOCOPP_EWORKSPACE);
            s_last = arrived == unsigned(c1 - c0 + 1);
            __threadfence();
        }
        if (!consumer_sync()) return false;
        if (s_last) {
            if (!merge_plane<T, D, G, W>(p, bg, c0, c1, int64_t(mt.b) * p.hq + mt.g * G, scratch, scratch_floats,
                                         consumer_sync, ctid, stage))
                return false;
        }
    }
    return consumer_sync();
}

template <typename T, int D, int G, int W, int STAGES, int CTAS_PER_SM, bool FUSED>
__global__ void __launch_bounds__((W + 1) * 32, CTAS_PER_SM)
decode_split_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                    const __grid_constant__ CUtensorMap tmK1, const __grid_constant__ CUtensorMap tmV1,
                    const DecodeParams p) {
    using S = DecodeShape<D, T, FUSED>;
    using L = DecodeSmem<T, D, G, W, STAGES, FUSED>;
    constexpr int TILE = S::TILE, TPW = L::TPW;

    extern __shared__ uint8_t smem_raw[];
    __shared__ int s_warp[32];
    __shared__ volatile int s_abort;
    __shared__ int s_cdone;
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* stage_mem = base;
    uint64_t* full_bar = reinterpret_cast<uint64_t*>(base + L::kBars);
    uint64_t* empty_bar = full_bar + STAGES;
    uint64_t* sync_bar = empty_bar + STAGES;  // consumer warps' merge rendezvous
    uint64_t* merge_bar = sync_bar + 1;       // the final merge's bulk copy
    TileMeta* meta = reinterpret_cast<TileMeta*>(base + L::kMeta);
    float* p_s = reinterpret_cast<float*>(base + L::kP);
    float* mg_m = reinterpret_cast<float*>(base + L::kMergeM);
    float* mg_l = reinterpret_cast<float*>(base + L::kMergeL);
    float* mg_o = reinterpret_cast<float*>(base + L::kMergeO);
    int* s_ts = reinterpret_cast<int*>(base + L::kTileStart);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], W);
        }
        mbar_init(sync_bar, W);
        mbar_init(merge_bar, 1);
        fence_mbar_init();
        s_abort = 0;
        s_cdone = 0;
    }
    // launched as a programmatic dependent: inputs may still be in flight
    // from the previous kernel until this wait returns
    griddep_wait();
    griddep_launch_dependents();
    __shared__ unsigned long long s_epoch;
    if (tid == 0) s_epoch = join_call(p.ws_gen, gridDim.x);
    tile_prefix<TILE>(p, s_ts, s_warp, blockDim.x);  // ends with a block-wide rendezvous
    const unsigned long long epoch = s_epoch;
    // sequences with no cached positions: zero output (CTA b mod grid writes it)
    for (int b = blockIdx.x; b < p.batch; b += p.num_ctas) {
        if (s_ts[b + 1] != s_ts[b]) continue;
        for (int idx = tid; idx < p.hq * D; idx += blockDim.x)
            emit<T, D>(p, int64_t(b) * p.hq + idx / D, idx % D, NEG_INF_F, 0.f, 0.f);
    }

    const SplitPlan sp = make_plan(p, s_ts, p.seg_units);
    const int2 range = plan_range(p, s_ts, sp, lane);
    const int start = range.x, end = range.y;
    if (start >= end) return;

    if (warp == W) {
        // ------------------------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tensormap(&tmK);
            prefetch_tensormap(&tmV);
            if constexpr (FUSED) {
                prefetch_tensormap(&tmK1);
                prefetch_tensormap(&tmV1);
            }
        }
        constexpr int NSB_MAX = 4;  // sub-boxes per tile when blocks are shorter than a tile
        const int nsb = TILE / p.boxr;
        int it = 0;
        int last_issued_it[STAGES];
#pragma unroll
        for (int s = 0; s < STAGES; ++s) last_issued_it[s] = -1;
        bool stop = false;
        for (int t0 = start; t0 < end && !stop; t0 += 32) {
            // lanes decode 32 upcoming tiles in parallel (block-table reads overlap)
            const int t = t0 + lane;
            int b = 0, g = 0, k = 0, len = 0, flags = 0;
            int rows[NSB_MAX] = {-1, -1, -1, -1};
            if (t < end) {
                int lo = 0, hi = p.batch;  // s_ts[lo] <= t < s_ts[hi]
                while (hi - lo > 1) {
                    const int mid = (lo + hi) >> 1;
                    if (s_ts[mid] <= t) lo = mid; else hi = mid;
                }
                b = lo;
                len = clamp_len(p.seq_lens, b, p.capacity);
                const int nt = ntiles_of(len, TILE);
                const int local = t - s_ts[b];
                g = local / nt;
                k = local - g * nt;
                const int plane0 = s_ts[b] + g * nt;
                if (t == start || k == 0) flags |= kFirst;
                if (t == end - 1 || k == nt - 1) flags |= kLast;
                if (plane0 >= start && plane0 + nt <= end) flags |= kWhole;
                if (p.block_table == nullptr) {
                    rows[0] = (b * p.hkv + g) * p.capacity + k * TILE;
                } else {
                    for (int s = 0; s < nsb; ++s) {
                        const int tok = k * TILE + s * p.boxr;
                        if (tok >= len) break;
                        const int blk = __ldg(p.block_table + int64_t(b) * p.mbps + tok / p.block_size);
                        if (blk < 0 || blk >= p.num_blocks) {
                            record_status(YOCOPP_EDEVICE_CHECK);
                            continue;
                        }
                        rows[s] = (blk * p.hkv + g) * p.block_size + tok % p.block_size;
                    }
                }
            }
            const int nthis = min(32, end - t0);
            for (int j = 0; j < nthis; ++j, ++it) {
                TileMeta m;
                m.b = __shfl_sync(0xffffffffu, b, j);
                m.g = __shfl_sync(0xffffffffu, g, j);
                m.k = __shfl_sync(0xffffffffu, k, j);
                m.len = __shfl_sync(0xffffffffu, len, j);
                m.flags = __shfl_sync(0xffffffffu, flags, j);
                m.pad = TILE;  // the tile size, for the plane's tile count at flush
                int r[NSB_MAX];
#pragma unroll
                for (int s = 0; s < NSB_MAX; ++s) r[s] = __shfl_sync(0xffffffffu, rows[s], j);
                const int stage = it % STAGES;
                const uint32_t parity = ((it / STAGES) & 1) ^ 1;
                int ok = 1;
                if (lane == 0) {
                    ok = mbar_wait(&empty_bar[stage], parity, p.wait_limit_ns) ? 1 : 0;
                    if (!ok) {
                        record_status(YOCOPP_ETIMEOUT);
                        s_abort = 1;
                    } else if (s_abort) {
                        ok = 0;
                    }
                }
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) {
                    stop = true;
                    break;
                }
                if (lane == 0) {
                    meta[stage] = m;
                    if (start + it != p.drop_tile) {
                        uint32_t nvalid = 0;
                        for (int s = 0; s < nsb; ++s) nvalid += r[s] >= 0 ? 1u : 0u;
                        const uint32_t bytes = nvalid * uint32_t(S::NBOX * p.boxr * 128 * S::NSRC);
                        mbar_arrive_expect_tx(&full_bar[stage], bytes);
                        uint8_t* kdst = stage_mem + size_t(stage) * S::STAGE_BYTES;
                        uint8_t* vdst = kdst + S::KV_BYTES;
                        for (int s = 0; s < nsb; ++s) {
                            if (r[s] < 0) continue;
#pragma unroll
                            for (int bx = 0; bx < S::NBOX; ++bx) {
                                const int off = bx * S::BOXB + s * p.boxr * 128;
                                tma_load_2d(kdst + off, &tmK, &full_bar[stage], bx * (128 / S::EB), r[s]);
                                tma_load_2d(vdst + off, &tmV, &full_bar[stage], bx * (128 / S::EB), r[s]);
                                if constexpr (FUSED) {
                                    tma_load_2d(kdst + 2 * S::KV_BYTES + off, &tmK1, &full_bar[stage],
                                                bx * (128 / S::EB), r[s]);
                                    tma_load_2d(kdst + 3 * S::KV_BYTES + off, &tmV1, &full_bar[stage],
                                                bx * (128 / S::EB), r[s]);
                                }
                            }
                        }
                        last_issued_it[stage] = it;
                    }
                }
                __syncwarp();
            }
        }
        // Stay until the consumer warps are done; if any of them gave up, wait
        // (bounded) for this CTA's copies still in flight before exiting.
        if (lane == 0) {
            const uint64_t t0 = globaltimer_ns();
            while (atomicAdd(&s_cdone, 0) < W && globaltimer_ns() - t0 <= p.wait_limit_ns) __nanosleep(256);
            if (s_abort) {
#pragma unroll
                for (int s = 0; s < STAGES; ++s)
                    if (last_issued_it[s] >= 0)
                        (void)mbar_wait(&full_bar[s], (last_issued_it[s] / STAGES) & 1, p.wait_limit_ns);
            }
        }
        return;
    }

    // ---------------------------------------------------------------------- consumers
    ConsumerWarp<T, D, G, W, FUSED> cw(warp, lane);
    cw.fk1 = make_float2(p.fa1k, p.fa1k);
    cw.fk2 = make_float2(p.fa2k, p.fa2k);
    cw.fv1 = make_float2(p.fa1v, p.fa1v);
    cw.fv2 = make_float2(p.fa2v, p.fa2v);
    __shared__ int s_last;
    float2* p2 = reinterpret_cast<float2*>(p_s) + warp * TPW * G;  // this warp's (p, p) pairs

    int nsync = 0;
    // bounded rendezvous of the W consumer warps (a named barrier could not time out);
    // every lane waits and the warp proceeds only if all lanes saw the phase complete
    auto consumer_sync = [&]() -> bool {
        __syncwarp();
        if (lane == 0) mbar_arrive(sync_bar);
        const bool ok = __all_sync(0xffffffffu, mbar_wait(sync_bar, nsync & 1, p.wait_limit_ns));
        ++nsync;
        return ok;
    };

    int snap_plane = -1;
    unsigned long long snap = 0;
    int it = 0;
    for (int t = start; t < end; ++t, ++it) {
        const int stage = it % STAGES;
        const uint32_t parity = (it / STAGES) & 1;
        const bool ready = !s_abort && mbar_wait(&full_bar[stage], parity, p.wait_limit_ns);
        if (!__all_sync(0xffffffffu, ready)) {
            record_status(YOCOPP_ETIMEOUT);
            s_abort = 1;
            break;
        }
        const TileMeta mt = meta[stage];
        const uint8_t* Kt = stage_mem + size_t(stage) * S::STAGE_BYTES;
        const uint8_t* Vt = Kt + S::KV_BYTES;
        if (tid == 0 && t == max(start, end - 3)) {  // the final plane's counter, read ahead
            snap_plane = mt.b * p.hkv + mt.g;
            snap = ld_relaxed_gpu(p.ws_cnt + snap_plane);
        }
        if (mt.flags & kFirst) cw.begin_segment(p, mt.b, mt.g);
        const int tok0 = mt.k * TILE + warp * TPW;  // first token of this warp's slice
        if (tok0 + TPW <= mt.len)
            cw.template tile<false>(Kt, Vt, p2, tok0, mt.len);
        else
            cw.template tile<true>(Kt, Vt, p2, tok0, mt.len);
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty_bar[stage]);

        if (mt.flags & kLast) {
            // ---- end of segment: merge the warps' states, emit output or a partial
            cw.stash(mg_m, mg_l, mg_o);
            // at the CTA's last tile the ring is free: a final merge may stage partials there
            const MergeStage ring{stage_mem, uint32_t(L::kStages), merge_bar};
            if (!flush_segment<T, D, G, W>(p, mt, tid, sp, s_ts, mg_m, mg_l, mg_o, p_s,
                                           int((L::kTileStart - L::kP) / sizeof(float)), consumer_sync, s_last,
                                           epoch, t == end - 1 ? &ring : nullptr,
                                           int((L::kMergeM - L::kP) / sizeof(float)), snap_plane, snap)) {
                record_status(YOCOPP_ETIMEOUT);
                s_abort = 1;
                break;
            }
        }
    }
    __syncwarp();
    if (lane == 0) atomicAdd(&s_cdone, 1);
}

// Merge R unnormalised partials [R][rows][D + 2] (o, m, l per row, as the
// partial mode writes them) into out [rows][D]: M = max_r m_r,
// out = sum_r 2^{m_r - M} o_r / sum_r 2^{m_r - M} l_r; rows with no tokens
// anywhere (all m = -inf) give 0.  One CTA per row, one thread per channel.
template <typename T, int D>
__global__ void __launch_bounds__(D) combine_parts_kernel(const float* parts, int nparts, int64_t rows, uint8_t* out) {
    const int64_t row = blockIdx.x;
    const int c = threadIdx.x;
    const int64_t stride = rows * (D + 2);
    float M = NEG_INF_F;
    for (int r = 0; r < nparts; ++r) M = fmaxf(M, parts[r * stride + row * (D + 2) + D]);
    float Ls = 0.f, O = 0.f;
    if (M != NEG_INF_F) {
        for (int r = 0; r < nparts; ++r) {
            const float* pr = parts + r * stride + row * (D + 2);
            const float f = exp2f(pr[D] - M);
            Ls += f * pr[D + 1];
            O += f * pr[c];
        }
    }
    write_out<T>(out, row * D + c, Ls > 0.f ? O / Ls : 0.f);
}

}  // namespace yocopp
