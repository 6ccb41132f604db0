// Split-K GQA decode attention with the query-group x key-tile scores on the
// 5th-generation tensor cores (tcgen05), bf16, head_dim 128.
//
// Same work decomposition, online softmax, value accumulation and segment
// merge as decode_split_kernel (decode_attn.cuh); only the score product
// moves: S^T = K_tile . Q_group^T is a [128 tokens] x [16 query rows] x [128
// channels] product, issued as eight tcgen05.mma (M = 128, N = 16, K = 16)
// by one thread into a 16-column accumulator in tensor memory.  The K tile
// and a 16-row block of q (the group's G heads plus the rows after them,
// which only produce unused columns) arrive by TMA with a 128-byte swizzle,
// which is the canonical K-major layout the MMA reads.  Two accumulators
// alternate between tiles.
//
// Warps: 0 = TMA producer, 1 = MMA issuer and tensor-memory owner,
// 2..5 = consumers, 6 = the L2 prefetch of the first tiles
// (prefetch_first_tiles), which runs before the programmatic wait and exits;
// the block-wide rendezvous of the others counts warps 0..5 only.  A warp may
// only read the tensor-memory lanes of its quadrant (warp index mod 4), so
// consumer warp w owns tile rows 32 (w mod 4) .. +31: one token per lane for
// the scores and the softmax, then (as in the CUDA-core kernel) lanes own
// 16-byte channel chunks for the value sum.  Every wait is bounded; the tensor
// memory is freed on every exit path after the MMAs in flight have completed.
#pragma once

#include "decode_attn.cuh"

namespace yocopp {

struct TcShape {
    static constexpr int D = 128, TILE = 128, ROWB = 256, NBOX = 2;
    static constexpr int BOXB = TILE * 128;                      // one 128-byte column box of a tile
    static constexpr int KV_BYTES = TILE * ROWB;                 // 32 KB
    static constexpr int QROWS = 16;                             // MMA N: query rows (heads, padded)
    static constexpr int QBOXB = QROWS * 128;                    // one column box of the q block
    static constexpr int Q_BYTES = NBOX * QBOXB;                 // 4 KB
    static constexpr int STAGE_BYTES = 2 * KV_BYTES + Q_BYTES;   // K, V, q
    static constexpr int W = 4;                                  // consumer warps
    static constexpr int TPW = 32;                               // tokens per consumer warp per tile
    static constexpr int CPR = 16, EPC = 8, TPI = 2;             // value phase layout (as the CUDA-core kernel)
    static constexpr int TMEM_COLS = 32;                         // two 16-column accumulators
    static constexpr uint32_t IDESC = umma_idesc_bf16(128, 16);
    static constexpr int NSB_MAX = 8;                            // sub-boxes per tile (block size 16)
    static constexpr int WORKERS = (W + 2) * 32;                 // producer, MMA and consumer warps
    static constexpr int THREADS = WORKERS + 32;                 // + the prefetch warp
};
static_assert(TcShape::STAGE_BYTES % 1024 == 0, "stage alignment");

template <int G, int STAGES>
struct TcSmem {
    using S = TcShape;
    __host__ __device__ static constexpr size_t up16(size_t x) { return (x + 15) & ~size_t(15); }
    static constexpr size_t kStages = size_t(STAGES) * S::STAGE_BYTES;
    static constexpr size_t kBars = kStages;  // full[S], empty[S], sfull[2], sempty[2], sync, merge
    static constexpr size_t kTmem = up16(kBars + (2 * STAGES + 6) * sizeof(uint64_t));
    static constexpr size_t kMeta = up16(kTmem + 16);
    static constexpr size_t kP = up16(kMeta + STAGES * sizeof(TileMeta));
    static constexpr size_t kMergeM = up16(kP + size_t(S::W) * S::TPW * G * sizeof(float2));
    static constexpr size_t kMergeL = up16(kMergeM + size_t(S::W) * G * sizeof(float));
    static constexpr size_t kMergeO = up16(kMergeL + size_t(S::W) * G * sizeof(float));
    static constexpr size_t kTileStart = up16(kMergeO + size_t(S::W) * G * S::D * sizeof(float));
    // after s_ts, for the batches the prefetch warp handles: its guess of s_ts
    __host__ __device__ static size_t guess_offset(int batch) { return up16(kTileStart + size_t(batch + 1) * sizeof(int)); }
    static size_t bytes(int batch) {
        return 1024 + guess_offset(batch) + (batch <= kGuessMaxBatch ? size_t(batch + 1) * sizeof(int) : 0);
    }
};

// One consumer warp: 32 token rows of every tile.
template <int G>
struct TcConsumerWarp {
    using S = TcShape;
    static constexpr int D = S::D, EPC = S::EPC, TPI = S::TPI, PV_IT = S::TPW / S::TPI;
    float2 acc[G][EPC / 2];
    float m_run[G];
    float l_lane[G];
    const int cw, qd, lane, pc, pslot, pbx, pcc;

    __device__ __forceinline__ TcConsumerWarp(int cw_, int qd_, int lane_)
        : cw(cw_), qd(qd_), lane(lane_), pc(lane_ % S::CPR), pslot(lane_ / S::CPR), pbx((lane_ % S::CPR) >> 3),
          pcc((lane_ % S::CPR) & 7) {}

    __device__ __forceinline__ void begin_segment() {
#pragma unroll
        for (int h = 0; h < G; ++h) {
            m_run[h] = NEG_INF_F;
            l_lane[h] = 0.f;
#pragma unroll
            for (int e = 0; e < EPC / 2; ++e) acc[h][e] = make_float2(0.f, 0.f);
        }
    }

    // sc: this lane's token's raw scores q.k for the G heads (from tensor memory).
    template <bool MASK>
    __device__ __forceinline__ void tile(const float (&sc)[4], const uint8_t* Vt, float2* p2, int tok0, int len,
                                         float qscale) {
        const int rbase = 32 * qd;
        float s[G];
#pragma unroll
        for (int h = 0; h < G; ++h) s[h] = (MASK && tok0 + lane >= len) ? NEG_INF_F : sc[h] * qscale;
        float mx[G];
#pragma unroll
        for (int h = 0; h < G; ++h) mx[h] = s[h];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
#pragma unroll
            for (int h = 0; h < G; ++h) mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], o));
        bool grow = false;
#pragma unroll
        for (int h = 0; h < G; ++h) grow |= mx[h] > m_run[h];
        if (grow) {
#pragma unroll
            for (int h = 0; h < G; ++h) {
                const float mnew = fmaxf(m_run[h], mx[h]);
                const float corr = mnew == NEG_INF_F ? 1.f : exp2f(m_run[h] - mnew);
                m_run[h] = mnew;
                l_lane[h] *= corr;
                const float2 c2 = make_float2(corr, corr);
#pragma unroll
                for (int e = 0; e < EPC / 2; ++e) acc[h][e] = fmul2(acc[h][e], c2);
            }
        }
        float pr[G];
#pragma unroll
        for (int h = 0; h < G; ++h) {
            pr[h] = (MASK && s[h] == NEG_INF_F) ? 0.f : exp2f(s[h] - m_run[h]);
            l_lane[h] += pr[h];
        }
        if constexpr (G >= 2) {
#pragma unroll
            for (int h = 0; h < G; h += 2)
                *reinterpret_cast<float4*>(p2 + lane * G + h) = make_float4(pr[h], pr[h], pr[h + 1], pr[h + 1]);
        } else {
            p2[lane] = make_float2(pr[0], pr[0]);
        }
        __syncwarp();
#pragma unroll 4
        for (int i2 = 0; i2 < PV_IT; ++i2) {
            const int tl = i2 * TPI + pslot;
            const int tk = rbase + tl;
            float2 vf[EPC / 2];
            load_pairs<__nv_bfloat16, false>(Vt + pbx * S::BOXB + tk * 128 + ((pcc ^ (tk & 7)) << 4), nullptr,
                                             make_float2(0.f, 0.f), make_float2(0.f, 0.f), vf);
            if (MASK && tok0 + tl >= len) {
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
        __syncwarp();
    }

    __device__ __forceinline__ void stash(float* mg_m, float* mg_l, float* mg_o) {
        float lsum[G];
#pragma unroll
        for (int h = 0; h < G; ++h) lsum[h] = l_lane[h];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
#pragma unroll
            for (int h = 0; h < G; ++h) lsum[h] += __shfl_xor_sync(0xffffffffu, lsum[h], o);
#pragma unroll
        for (int h = 0; h < G; ++h)
#pragma unroll
            for (int e = 0; e < EPC / 2; ++e) {
                acc[h][e].x += __shfl_xor_sync(0xffffffffu, acc[h][e].x, 16);
                acc[h][e].y += __shfl_xor_sync(0xffffffffu, acc[h][e].y, 16);
            }
#pragma unroll
        for (int h = 0; h < G; ++h) {
            if (lane == 0) {
                mg_m[cw * G + h] = m_run[h];
                mg_l[cw * G + h] = lsum[h];
            }
            if (lane < S::CPR) {
#pragma unroll
                for (int e = 0; e < EPC / 2; ++e)
                    *reinterpret_cast<float2*>(mg_o + (cw * G + h) * D + lane * EPC + 2 * e) = acc[h][e];
            }
        }
    }
};

#ifndef YOCOPP_DECODE_PREFETCH_TILES
#define YOCOPP_DECODE_PREFETCH_TILES 2  // tiles per CTA prefetched into L2 before the programmatic wait
#endif

template <int G, int STAGES>
__global__ void __launch_bounds__(TcShape::THREADS, 1)
decode_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                 const __grid_constant__ CUtensorMap tmQ, const DecodeParams p) {
    using S = TcShape;
    using L = TcSmem<G, STAGES>;
    constexpr int TILE = S::TILE, W = S::W;
    static_assert(G == 1 || G == 2 || G == 4, "group size");

    extern __shared__ uint8_t smem_raw[];
    __shared__ int s_warp[32];
    __shared__ volatile int s_abort;
    __shared__ int s_cdone;
    __shared__ int s_last;
    // the call's epoch: taken by an otherwise idle lane of the MMA warp (its atomics are
    // round trips to L2) while the first tiles load; the consumers need it at their first flush
    __shared__ unsigned long long s_epoch;
    __shared__ volatile int s_epoch_ready;
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* stage_mem = base;
    uint64_t* full_bar = reinterpret_cast<uint64_t*>(base + L::kBars);
    uint64_t* empty_bar = full_bar + STAGES;
    uint64_t* sfull_bar = empty_bar + STAGES;   // accumulator b holds a finished score tile
    uint64_t* sempty_bar = sfull_bar + 2;       // accumulator b has been read
    uint64_t* sync_bar = sempty_bar + 2;        // consumer warps' merge rendezvous
    uint64_t* merge_bar = sync_bar + 1;         // the final merge's bulk copy
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + L::kTmem);
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
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sfull_bar[b], 1);
            mbar_init(&sempty_bar[b], W);
        }
        mbar_init(sync_bar, W);
        mbar_init(merge_bar, 1);
        fence_mbar_init();
        s_abort = 0;
        s_cdone = 0;
        s_epoch_ready = 0;
        prefetch_tensormap(&tmK);
        prefetch_tensormap(&tmV);
        prefetch_tensormap(&tmQ);
    }

    if (warp == W + 2) {
        // ---------------------------------------------- the prefetch, before the wait
        if (YOCOPP_DECODE_PREFETCH_TILES > 0 && p.prefetch && p.batch <= kGuessMaxBatch)
            prefetch_first_tiles<TILE, S::NBOX, S::NSB_MAX>(
                p, &tmK, &tmV, reinterpret_cast<int*>(base + L::guess_offset(p.batch)), YOCOPP_DECODE_PREFETCH_TILES,
                lane);
        return;
    }
    // tensor memory needs no input: take it while the previous kernel may still run
    if (warp == 1) {
        tmem_alloc(tmem_slot, S::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    griddep_wait();
    griddep_launch_dependents();
    tile_prefix<TILE>(p, s_ts, s_warp, S::WORKERS);  // ends with a rendezvous of warps 0..W+1
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    for (int b = blockIdx.x; b < p.batch; b += p.num_ctas) {
        if (s_ts[b + 1] != s_ts[b]) continue;
        for (int idx = tid; idx < p.hq * S::D; idx += S::WORKERS)
            emit<__nv_bfloat16, S::D>(p, int64_t(b) * p.hq + idx / S::D, idx % S::D, NEG_INF_F, 0.f, 0.f);
    }
    const SplitPlan sp = make_plan(p, s_ts, p.seg_units);
    const int2 range = plan_range(p, s_ts, sp, lane);
    const int start = range.x, end = range.y;
    if (start >= end) {
        if (tid == 0) (void)join_call(p.ws_gen, gridDim.x);  // every CTA joins the call
        if (warp == 1) tmem_dealloc(tmem, S::TMEM_COLS);
        return;
    }

    if (warp == 0) {
        // ------------------------------------------------------------------ producer
        // one tile's loads into a stage: K and V sub-boxes at rows r (-1: none), the group's q block
        const int nsb = TILE / p.boxr;
        auto issue_tile = [&](int stage, const int* r, int b, int g, uint64_t* bar) {
            uint32_t nvalid = 0;
            for (int s = 0; s < nsb; ++s) nvalid += r[s] >= 0 ? 1u : 0u;
            mbar_arrive_expect_tx(bar, nvalid * uint32_t(S::NBOX * p.boxr * 128 * 2) + uint32_t(S::Q_BYTES));
            uint8_t* kdst = stage_mem + size_t(stage) * S::STAGE_BYTES;
            uint8_t* vdst = kdst + S::KV_BYTES;
            uint8_t* qdst = vdst + S::KV_BYTES;
            for (int s = 0; s < nsb; ++s) {
                if (r[s] < 0) continue;
#pragma unroll
                for (int bx = 0; bx < S::NBOX; ++bx) {
                    const int off = bx * S::BOXB + s * p.boxr * 128;
                    tma_load_2d(kdst + off, &tmK, bar, bx * 64, r[s]);
                    tma_load_2d(vdst + off, &tmV, bar, bx * 64, r[s]);
                }
            }
#pragma unroll
            for (int bx = 0; bx < S::NBOX; ++bx) tma_load_2d(qdst + bx * S::QBOXB, &tmQ, bar, bx * 64, b * p.hq + g * G);
        };
        int it = 0;
        int last_issued_it[STAGES];
#pragma unroll
        for (int s = 0; s < STAGES; ++s) last_issued_it[s] = -1;
        bool stop = false;
        for (int t0 = start; t0 < end && !stop; t0 += 32) {
            const int t = t0 + lane;
            int b = 0, g = 0, k = 0, len = 0, flags = 0;
            int rows[S::NSB_MAX];
#pragma unroll
            for (int s = 0; s < S::NSB_MAX; ++s) rows[s] = -1;
            if (t < end) {
                int lo = 0, hi = p.batch;
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
#pragma unroll
                    for (int s = 0; s < S::NSB_MAX; ++s) {
                        const int tok = k * TILE + s * p.boxr;
                        if (s >= nsb || tok >= len) continue;
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
                m.pad = TILE;
                int r[S::NSB_MAX];
#pragma unroll
                for (int s = 0; s < S::NSB_MAX; ++s) r[s] = __shfl_sync(0xffffffffu, rows[s], j);
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
                        issue_tile(stage, r, m.b, m.g, &full_bar[stage]);
                        last_issued_it[stage] = it;
                    }
                }
                __syncwarp();
            }
        }
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

    if (warp == 1) {
        // ------------------------------------------------------------- MMA issuer
        int last_it[2] = {-1, -1};
        if (lane == 1) {
            s_epoch = join_call(p.ws_gen, gridDim.x);
            __threadfence_block();
            s_epoch_ready = 1;
        }
        if (lane == 0) {
            int it = 0;
            for (int t = start; t < end; ++t, ++it) {
                const int stage = it % STAGES;
                const int buf = it & 1;
                const bool ok = !s_abort && mbar_wait(&full_bar[stage], (it / STAGES) & 1, p.wait_limit_ns) &&
                                mbar_wait(&sempty_bar[buf], ((it >> 1) & 1) ^ 1, p.wait_limit_ns);
                if (!ok) {
                    record_status(YOCOPP_ETIMEOUT);
                    s_abort = 1;
                    break;
                }
                tc_fence_after();
                const uint32_t kaddr = smem_addr(stage_mem + size_t(stage) * S::STAGE_BYTES);
                const uint32_t qaddr = kaddr + 2 * S::KV_BYTES;
#pragma unroll
                for (int kk = 0; kk < S::D / 16; ++kk) {
                    const uint32_t koff = uint32_t((kk >> 2) * S::BOXB + (kk & 3) * 32);
                    const uint32_t qoff = uint32_t((kk >> 2) * S::QBOXB + (kk & 3) * 32);
                    umma_bf16(tmem + uint32_t(buf * 16), umma_desc_sw128(kaddr + koff), umma_desc_sw128(qaddr + qoff),
                              S::IDESC, kk > 0 ? 1u : 0u);
                }
                umma_commit(&sfull_bar[buf]);
                last_it[buf] = it;
            }
            // wait until the consumers are done with tensor memory; after an abort, also
            // until the MMAs still in flight have completed
            const uint64_t t0 = globaltimer_ns();
            while (atomicAdd(&s_cdone, 0) < W && globaltimer_ns() - t0 <= p.wait_limit_ns) __nanosleep(256);
            if (s_abort) {
                for (int b2 = 0; b2 < 2; ++b2)
                    if (last_it[b2] >= 0) (void)mbar_wait(&sfull_bar[b2], (last_it[b2] >> 1) & 1, p.wait_limit_ns);
            }
        }
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, S::TMEM_COLS);
        return;
    }

    // ---------------------------------------------------------------------- consumers
    const int cw_idx = warp - 2;          // 0..3
    const int ctid = tid - 64;            // consumer thread index
    TcConsumerWarp<G> cw(cw_idx, warp & 3, lane);
    float2* p2 = reinterpret_cast<float2*>(p_s) + cw_idx * S::TPW * G;
    const uint32_t my_lanes = uint32_t(32 * (warp & 3)) << 16;

    int nsync = 0;
    auto consumer_sync = [&]() -> bool {
        __syncwarp();
        if (lane == 0) mbar_arrive(sync_bar);
        const bool ok = __all_sync(0xffffffffu, mbar_wait(sync_bar, nsync & 1, p.wait_limit_ns));
        ++nsync;
        return ok;
    };

    unsigned long long epoch = 0;  // epochs start at 1
    int snap_plane = -1;
    unsigned long long snap = 0;
    int it = 0;
    for (int t = start; t < end; ++t, ++it) {
        const int stage = it % STAGES;
        const int buf = it & 1;
        const bool ready = !s_abort && mbar_wait(&full_bar[stage], (it / STAGES) & 1, p.wait_limit_ns) &&
                           mbar_wait(&sfull_bar[buf], (it >> 1) & 1, p.wait_limit_ns);
        if (!__all_sync(0xffffffffu, ready)) {
            record_status(YOCOPP_ETIMEOUT);
            s_abort = 1;
            break;
        }
        const TileMeta mt = meta[stage];
        if (ctid == 0 && t == max(start, end - 3)) {  // the final plane's counter, read ahead
            snap_plane = mt.b * p.hkv + mt.g;
            snap = ld_relaxed_gpu(p.ws_cnt + snap_plane);
        }
        if (mt.flags & kFirst) cw.begin_segment();
        tc_fence_after();
        float sc[4];
        tmem_ld4(tmem + my_lanes + uint32_t(buf * 16), sc);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sempty_bar[buf]);

        const uint8_t* Vt = stage_mem + size_t(stage) * S::STAGE_BYTES + S::KV_BYTES;
        const int tok0 = mt.k * TILE + 32 * (warp & 3);
        if (tok0 + 32 <= mt.len)
            cw.template tile<false>(sc, Vt, p2, tok0, mt.len, p.qscale);
        else
            cw.template tile<true>(sc, Vt, p2, tok0, mt.len, p.qscale);
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty_bar[stage]);

        if (mt.flags & kLast) {
            if (epoch == 0) {  // first flush: the epoch was taken long ago
                const uint64_t t0 = globaltimer_ns();
                while (!s_epoch_ready && globaltimer_ns() - t0 <= p.wait_limit_ns) __nanosleep(32);
                if (!__all_sync(0xffffffffu, s_epoch_ready != 0)) {
                    record_status(YOCOPP_ETIMEOUT);
                    s_abort = 1;
                    break;
                }
                __threadfence_block();
                epoch = s_epoch;
            }
            cw.stash(mg_m, mg_l, mg_o);
            // at the CTA's last tile the ring is free (every load and product that used it
            // has completed): a final merge may stage partials there
            const MergeStage ring{stage_mem, uint32_t(L::kStages), merge_bar};
            if (!flush_segment<__nv_bfloat16, S::D, G, W>(p, mt, ctid, sp, s_ts, mg_m, mg_l, mg_o, p_s,
                                                          int((L::kTileStart - L::kP) / sizeof(float)),
                                                          consumer_sync, s_last, epoch,
                                                          t == end - 1 ? &ring : nullptr,
                                                          int((L::kMergeM - L::kP) / sizeof(float)), snap_plane,
                                                          snap)) {
                record_status(YOCOPP_ETIMEOUT);
                s_abort = 1;
                break;
            }
        }
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) atomicAdd(&s_cdone, 1);
}

}  // namespace yocopp
