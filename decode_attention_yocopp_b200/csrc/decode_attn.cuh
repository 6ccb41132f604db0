// Split-K GQA decode attention over the shared cross-decoder cache.
//
// You Only Cache Once (abstract): the cross-decoder reuses the self-decoder's
// cache through cross-attention.  YOCO++ section 2: every upper-half layer
// reads the middle layer's composed cache (K'_{L/2}, V'_{L/2}); section 3
// ("efficiency analysis"): decoding reads exactly one KV set per layer, so a
// decode step is bound by HBM bandwidth on these reads.
//
// Work decomposition.  The (sequence, kv-head) planes are cut into TILE-token
// tiles and flattened in (b, g, tile) order.  A persistent grid of one CTA per
// SM takes equal contiguous ranges of that list, so any length mix is
// balanced to within one tile and each CTA streams contiguous K/V.  A CTA
// keeps online-softmax state for the (b, g) "segment" it is in; at the end of
// a segment it writes either the final output (segment = the whole plane) or
// an unnormalised partial (max, sum of exponentials, weighted value sum) to a
// workspace slot; the combine kernel merges partials of planes that span
// several CTAs with an exact log-sum-exp.
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
    int32_t* ws_tile_start;      // [batch + 1]
    float* ws_m;                 // [slots][G]
    float* ws_l;                 // [slots][G]
    float* ws_o;                 // [slots][G][D]
    float qscale;                // softmax scale * log2(e)
    int32_t batch, hkv, hq, capacity, block_size, mbps, num_blocks, boxr;
    int32_t num_ctas;
    int32_t drop_tile;           // testing: a tile whose load is never issued (-1: none)
    uint64_t wait_limit_ns;
};

struct TileMeta {
    int32_t b, g, k, len, flags, pad;
};
enum : int32_t { kFirst = 1, kLast = 2, kWhole = 4 };

template <int D, typename T>
struct DecodeShape {
    static constexpr int EB = sizeof(T);
    static constexpr int ROWB = D * EB;                   // bytes per (token, head) row
    static constexpr int TILE = ROWB <= 256 ? 64 : 32;    // tokens per pipeline tile
    static constexpr int NBOX = ROWB / 128;               // 128-byte swizzle boxes per row
    static constexpr int BOXB = TILE * 128;               // bytes of one box column of a tile
    static constexpr int KV_BYTES = TILE * ROWB;          // one K (or V) tile
    static constexpr int STAGE_BYTES = 2 * KV_BYTES;
    static constexpr int CPR = ROWB / 16;                 // 16-byte chunks per row
    static constexpr int CPL = CPR / 8;                   // score phase: chunks per lane
    static constexpr int EPC = 16 / EB;                   // elements per chunk
    static constexpr int TPI = 32 / CPR;                  // value phase: tokens per warp step
};

__device__ __forceinline__ int ntiles_of(int len, int tile) { return (len + tile - 1) / tile; }

__device__ __forceinline__ int clamp_len(const int32_t* lens, int b, int cap) {
    int len = __ldg(lens + b);
    return len < 0 ? 0 : (len > cap ? cap : len);
}

// Block-wide exclusive prefix of tiles per sequence (x kv heads) into s_ts[0..batch].
template <int TILE>
__device__ void tile_prefix(const DecodeParams& p, int* s_ts, int* s_warp) {
    const int nthr = blockDim.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
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
    __syncthreads();
    if (warp == 0) {
        int v = lane < (nthr >> 5) ? s_warp[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, v, o);
            if (lane >= o) v += y;
        }
        s_warp[lane] = v;
    }
    __syncthreads();
    int excl = x - sum + (warp > 0 ? s_warp[warp - 1] : 0);
    for (int b = b0; b < b1; ++b) {
        s_ts[b] = excl;
        excl += ntiles_of(clamp_len(p.seq_lens, b, p.capacity), TILE) * p.hkv;
    }
    if (tid == nthr - 1) s_ts[p.batch] = excl;
    __syncthreads();
}

template <typename T, int D, int G, int W, int STAGES>
struct DecodeSmem {
    using S = DecodeShape<D, T>;
    static constexpr int TPW = S::TILE / W;
    static constexpr size_t up16(size_t x) { return (x + 15) & ~size_t(15); }
    static constexpr size_t kStages = size_t(STAGES) * S::STAGE_BYTES;      // 1024-aligned ring
    static constexpr size_t kBars = kStages;                                 // full[S], empty[S], sync
    static constexpr size_t kMeta = up16(kBars + (2 * STAGES + 1) * sizeof(uint64_t));
    static constexpr size_t kP = up16(kMeta + STAGES * sizeof(TileMeta));
    static constexpr size_t kMergeM = up16(kP + size_t(W) * TPW * G * sizeof(float));
    static constexpr size_t kMergeL = up16(kMergeM + size_t(W) * G * sizeof(float));
    static constexpr size_t kMergeO = up16(kMergeL + size_t(W) * G * sizeof(float));
    static constexpr size_t kTileStart = up16(kMergeO + size_t(W) * G * D * sizeof(float));
    static size_t bytes(int batch) { return 1024 + kTileStart + size_t(batch + 1) * sizeof(int); }
};

template <typename T, int D, int G, int W, int STAGES>
__global__ void __launch_bounds__((W + 1) * 32, 1)
decode_split_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                    const DecodeParams p) {
    using S = DecodeShape<D, T>;
    using L = DecodeSmem<T, D, G, W, STAGES>;
    constexpr int TILE = S::TILE, TPW = L::TPW, CPR = S::CPR, CPL = S::CPL, EPC = S::EPC, TPI = S::TPI;
    constexpr int QK_IT = TPW / 4;
    constexpr int PV_IT = TPW / TPI;
    constexpr int HL = 8 / G;  // lanes holding one head's score after the reduce-scatter
    static_assert(G == 1 || G == 2 || G == 4, "group size");
    static_assert(TPW % 4 == 0 && TPW % TPI == 0, "tile split");

    extern __shared__ uint8_t smem_raw[];
    __shared__ int s_warp[32];
    __shared__ volatile int s_abort;
    __shared__ int s_cdone;
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* stage_mem = base;
    uint64_t* full_bar = reinterpret_cast<uint64_t*>(base + L::kBars);
    uint64_t* empty_bar = full_bar + STAGES;
    uint64_t* sync_bar = empty_bar + STAGES;  // consumer warps' merge rendezvous
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
        fence_mbar_init();
        s_abort = 0;
        s_cdone = 0;
    }
    tile_prefix<TILE>(p, s_ts, s_warp);  // ends with __syncthreads()
    if (blockIdx.x == 0)
        for (int b = tid; b <= p.batch; b += blockDim.x) p.ws_tile_start[b] = s_ts[b];

    const int total = s_ts[p.batch];
    const int tpc = (total + p.num_ctas - 1) / p.num_ctas;
    const int start = min(int(blockIdx.x) * tpc, total);
    const int end = min(start + tpc, total);
    if (start >= end) return;

    if (warp == W) {
        // ------------------------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tensormap(&tmK);
            prefetch_tensormap(&tmV);
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
                m.pad = 0;
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
                        const uint32_t bytes = nvalid * uint32_t(S::NBOX * p.boxr * 128 * 2);
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
    const int j4 = lane >> 3;        // score phase: token slot within a step of 4
    const int r8 = lane & 7;         // score phase: lane within the token's 8
    const int hr = r8 / HL;          // head this lane's score belongs to
    const int pc = lane % CPR;       // value phase: channel chunk owned
    const int pslot = lane / CPR;    // value phase: token slot within a step
    const int pbx = pc >> 3, pcc = pc & 7;

    float2 q2[G][CPL * EPC / 2];
    float2 acc[G][EPC / 2];
    float m_run[G];
    float l_part = 0.f;
    const float NEG_INF = -INFINITY;

    int nsync = 0;
    // bounded rendezvous of the W consumer warps (a named barrier could not time out)
    // (every lane waits; the warp proceeds only if all lanes saw the phase complete)
    auto consumer_sync = [&]() -> bool {
        __syncwarp();
        if (lane == 0) mbar_arrive(sync_bar);
        const bool ok = __all_sync(0xffffffffu, mbar_wait(sync_bar, nsync & 1, p.wait_limit_ns));
        ++nsync;
        return ok;
    };

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

        if (mt.flags & kFirst) {
            // new (sequence, kv-head) segment: reset state, load the group's queries
#pragma unroll
            for (int h = 0; h < G; ++h) {
                m_run[h] = NEG_INF;
#pragma unroll
                for (int e = 0; e < EPC / 2; ++e) acc[h][e] = make_float2(0.f, 0.f);
                const uint8_t* qrow = p.q + (int64_t(mt.b) * p.hq + mt.g * G + h) * S::ROWB;
#pragma unroll
                for (int jb = 0; jb < CPL; ++jb) {
                    const uint4 v = ld_stream(qrow + (r8 + 8 * jb) * 16);
                    const uint32_t* w = reinterpret_cast<const uint32_t*>(&v);
                    if constexpr (S::EB == 2) {
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            float2 f = bf16x2_to_float2(w[e]);
                            q2[h][jb * 4 + e] = make_float2(f.x * p.qscale, f.y * p.qscale);
                        }
                    } else {
                        q2[h][jb * 2 + 0] = make_float2(__uint_as_float(w[0]) * p.qscale, __uint_as_float(w[1]) * p.qscale);
                        q2[h][jb * 2 + 1] = make_float2(__uint_as_float(w[2]) * p.qscale, __uint_as_float(w[3]) * p.qscale);
                    }
                }
            }
            l_part = 0.f;
        }

        // ---- scores: s = (q * scale * log2 e) . k for this warp's TPW tokens
        float s[QK_IT];
#pragma unroll
        for (int i = 0; i < QK_IT; ++i) {
            const int row = warp * TPW + i * 4 + j4;
            float2 part[G];
#pragma unroll
            for (int h = 0; h < G; ++h) part[h] = make_float2(0.f, 0.f);
#pragma unroll
            for (int jb = 0; jb < CPL; ++jb) {
                const uint4 kv = *reinterpret_cast<const uint4*>(Kt + jb * S::BOXB + row * 128 + ((r8 ^ (row & 7)) << 4));
                const uint32_t* w = reinterpret_cast<const uint32_t*>(&kv);
                if constexpr (S::EB == 2) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 kf = bf16x2_to_float2(w[e]);
#pragma unroll
                        for (int h = 0; h < G; ++h) part[h] = ffma2(q2[h][jb * 4 + e], kf, part[h]);
                    }
                } else {
                    const float2 k0 = make_float2(__uint_as_float(w[0]), __uint_as_float(w[1]));
                    const float2 k1 = make_float2(__uint_as_float(w[2]), __uint_as_float(w[3]));
#pragma unroll
                    for (int h = 0; h < G; ++h) {
                        part[h] = ffma2(q2[h][jb * 2 + 0], k0, part[h]);
                        part[h] = ffma2(q2[h][jb * 2 + 1], k1, part[h]);
                    }
                }
            }
            float v[G];
#pragma unroll
            for (int h = 0; h < G; ++h) v[h] = part[h].x + part[h].y;
            // reduce-scatter over the token's 8 lanes: lane r ends with head r / HL
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
            const int tok = mt.k * TILE + row;
            s[i] = tok < mt.len ? sc : NEG_INF;
        }

        // ---- online softmax update (log2 domain)
        float mloc = s[0];
#pragma unroll
        for (int i = 1; i < QK_IT; ++i) mloc = fmaxf(mloc, s[i]);
        mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, 8));
        mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, 16));
        float corr[G];
        float m_own = NEG_INF, corr_own = 1.f;
#pragma unroll
        for (int h = 0; h < G; ++h) {
            const float mt_h = __shfl_sync(0xffffffffu, mloc, h * HL);
            const float mnew = fmaxf(m_run[h], mt_h);
            corr[h] = mnew == NEG_INF ? 1.f : exp2f(m_run[h] - mnew);
            m_run[h] = mnew;
            if (h == hr) {
                m_own = mnew;
                corr_own = corr[h];
            }
        }
        l_part *= corr_own;
#pragma unroll
        for (int i = 0; i < QK_IT; ++i) {
            const float pr = s[i] == NEG_INF ? 0.f : exp2f(s[i] - m_own);
            l_part += pr;
            if (r8 % HL == 0) p_s[(warp * TPW + i * 4 + j4) * G + hr] = pr;
        }
#pragma unroll
        for (int h = 0; h < G; ++h) {
            const float2 c2 = make_float2(corr[h], corr[h]);
#pragma unroll
            for (int e = 0; e < EPC / 2; ++e) acc[h][e] = fmul2(acc[h][e], c2);
        }
        __syncwarp();

        // ---- values: acc[h] += p[h] * v over this warp's tokens
#pragma unroll
        for (int i2 = 0; i2 < PV_IT; ++i2) {
            const int tk = warp * TPW + i2 * TPI + pslot;
            uint4 vv = *reinterpret_cast<const uint4*>(Vt + pbx * S::BOXB + tk * 128 + ((pcc ^ (tk & 7)) << 4));
            if (mt.k * TILE + tk >= mt.len) vv = make_uint4(0u, 0u, 0u, 0u);  // never read past the sequence
            float pv[G];
            if constexpr (G == 4) {
                const float4 t4 = *reinterpret_cast<const float4*>(p_s + tk * 4);
                pv[0] = t4.x; pv[1] = t4.y; pv[2] = t4.z; pv[3] = t4.w;
            } else if constexpr (G == 2) {
                const float2 t2 = *reinterpret_cast<const float2*>(p_s + tk * 2);
                pv[0] = t2.x; pv[1] = t2.y;
            } else {
                pv[0] = p_s[tk];
            }
            const uint32_t* w = reinterpret_cast<const uint32_t*>(&vv);
            float2 vf[EPC / 2];
            if constexpr (S::EB == 2) {
#pragma unroll
                for (int e = 0; e < 4; ++e) vf[e] = bf16x2_to_float2(w[e]);
            } else {
                vf[0] = make_float2(__uint_as_float(w[0]), __uint_as_float(w[1]));
                vf[1] = make_float2(__uint_as_float(w[2]), __uint_as_float(w[3]));
            }
#pragma unroll
            for (int h = 0; h < G; ++h) {
                const float2 ph = make_float2(pv[h], pv[h]);
#pragma unroll
                for (int e = 0; e < EPC / 2; ++e) acc[h][e] = ffma2(ph, vf[e], acc[h][e]);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty_bar[stage]);

        if (mt.flags & kLast) {
            // ---- end of segment: merge the warps' states, emit output or a partial
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
            if (!consumer_sync()) {
                record_status(YOCOPP_ETIMEOUT);
                s_abort = 1;
                break;
            }
            const int slot = mt.b * p.hkv + mt.g + int(blockIdx.x);
            for (int idx = tid; idx < G * D; idx += W * 32) {
                const int h = idx / D, c = idx % D;
                float M = NEG_INF;
#pragma unroll
                for (int w2 = 0; w2 < W; ++w2) M = fmaxf(M, mg_m[w2 * G + h]);
                float Ls = 0.f, O = 0.f;
                if (M != NEG_INF) {
#pragma unroll
                    for (int w2 = 0; w2 < W; ++w2) {
                        const float f = exp2f(mg_m[w2 * G + h] - M);
                        Ls += f * mg_l[w2 * G + h];
                        O += f * mg_o[(w2 * G + h) * D + c];
                    }
                }
                if (mt.flags & kWhole) {
                    const float y = Ls > 0.f ? O / Ls : 0.f;
                    const int64_t oi = (int64_t(mt.b) * p.hq + mt.g * G + h) * D + c;
                    if constexpr (S::EB == 2)
                        reinterpret_cast<__nv_bfloat16*>(p.out)[oi] = __float2bfloat16_rn(y);
                    else
                        reinterpret_cast<float*>(p.out)[oi] = y;
                } else {
                    p.ws_o[(int64_t(slot) * G + h) * D + c] = O;
                    if (c == 0) {
                        p.ws_m[int64_t(slot) * G + h] = M;
                        p.ws_l[int64_t(slot) * G + h] = Ls;
                    }
                }
            }
            if (!consumer_sync()) {
                record_status(YOCOPP_ETIMEOUT);
                s_abort = 1;
                break;
            }
        }
    }
    __syncwarp();
    if (lane == 0) atomicAdd(&s_cdone, 1);
}

// Merge the partials of planes that span several CTAs; zero planes with no tokens.
template <typename T, int D, int G>
__global__ void __launch_bounds__(128) decode_combine_kernel(const DecodeParams p) {
    using S = DecodeShape<D, T>;
    const int bg = blockIdx.x;
    const int b = bg / p.hkv, g = bg % p.hkv;
    const int len = clamp_len(p.seq_lens, b, p.capacity);
    const int nt = ntiles_of(len, S::TILE);
    const int64_t obase = (int64_t(b) * p.hq + g * G) * D;
    if (nt == 0) {
        for (int idx = threadIdx.x; idx < G * D; idx += blockDim.x) {
            if constexpr (S::EB == 2)
                reinterpret_cast<__nv_bfloat16*>(p.out)[obase + idx] = __float2bfloat16_rn(0.f);
            else
                reinterpret_cast<float*>(p.out)[obase + idx] = 0.f;
        }
        return;
    }
    const int total = p.ws_tile_start[p.batch];
    const int tpc = (total + p.num_ctas - 1) / p.num_ctas;
    const int first = p.ws_tile_start[b] + g * nt;
    const int c0 = first / tpc, c1 = (first + nt - 1) / tpc;
    if (c0 == c1) return;  // the plane was finished inside one CTA
    for (int idx = threadIdx.x; idx < G * D; idx += blockDim.x) {
        const int h = idx / D, c = idx % D;
        float M = -INFINITY;
        for (int cta = c0; cta <= c1; ++cta) M = fmaxf(M, p.ws_m[int64_t(bg + cta) * G + h]);
        float Ls = 0.f, O = 0.f;
        for (int cta = c0; cta <= c1; ++cta) {
            const int64_t sl = bg + cta;
            const float f = exp2f(p.ws_m[sl * G + h] - M);
            Ls += f * p.ws_l[sl * G + h];
            O += f * p.ws_o[(sl * G + h) * D + c];
        }
        const float y = Ls > 0.f ? O / Ls : 0.f;
        if constexpr (S::EB == 2)
            reinterpret_cast<__nv_bfloat16*>(p.out)[obase + idx] = __float2bfloat16_rn(y);
        else
            reinterpret_cast<float*>(p.out)[obase + idx] = y;
    }
}

}  // namespace yocopp
