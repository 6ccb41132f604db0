// Causal prefill attention of a self-decoder layer over its own (composed)
// cache, with both products on the tcgen05 tensor cores.
//
// YOCO++: Enhancing YOCO with KV Residual Connections, section 2 (cache
// strategy: each self-decoder layer caches its composed K'_i, V'_i) and
// section 3 (prefill is compute-bound, and the composition adds only a little
// I/O to it).  The composition runs first as yocopp_compose_append, an HBM
// stream that writes the composed rows once; this kernel then attends, for
// query row j of sequence b (cache position p_b + j) and query head h, over
// cache positions [0, p_b + j] of KV head g = h / (hq / hkv):
//   out[b,j,h] = sum_u softmax_u(scale q . K'_u) V'_u.
//
// Work unit: one CTA per (sequence, 128-row query tile, pair of query heads
// of one KV head); the CTAs of one KV head plane run together, heaviest query
// tiles first.  The two heads ("a" and "b")
// share every K/V tile the CTA loads, which halves the K/V traffic per FLOP
// (a lone head per CTA streams 64 KB of K/V per 8.4 MFLOP, more than L2 can
// feed every SM at tensor-core speed).  With an odd group size each CTA takes
// one head.
//
// Tensor memory (512 columns): S_a, S_b (128 x 128 fp32 each) and O_a, O_b.
// Per key tile t and head x:
//   S_x = Q_x K^T  eight tcgen05.mma (M = 128 queries, N = 128 keys, K = 16
//                  channels), Q and K K-major from their TMA tiles;
//   softmax        one thread per query row: masks keys past its position,
//                  forms P = 2^(s - m) (its row sum taken over the bf16 values
//                  the product uses) against a reference maximum m that
//                  moves only when the row maximum exceeds it by more than 8
//                  (then O_x and the row sum are rescaled), so P <= 2^8 and
//                  rescales are rare; P is written as bf16 into the first 64
//                  columns of S_x (two keys per column), where the next
//                  product reads it;
//   O_x += P V     eight tcgen05.mma (M = 128, N = 128 channels, K = 16 keys)
//                  with P from tensor memory and V MN-major from its TMA tile.
// The tensor pipe runs PV_a(t), QK_a(t+1), PV_b(t), QK_b(t+1): while one
// head's softmax works, the other head's products run.  K and V stream
// through separate two-slot rings, each refilled by its own producer lane as
// soon as the last product reading the slot completes.
//
// prefill_tc_kernel<true> (yocopp_prefill_compose_attn) also composes the rows
// it attends over, in the same launch: composition CTAs placed ahead of the
// attention CTAs that read their rows, per-tile flags in the caller's
// workspace (see the comment above the kernel).
//
// Warps: 0 = TMA producer (lane 0: Q and K, lane 1: V), 1 = MMA issuer and
// tensor-memory owner, 2..5 = softmax and epilogue of head a, 6..9 = head b
// (warp w reads TMEM lanes 32 (w mod 4) .. + 31).  Every wait is bounded; on
// a timeout the kernel records YOCOPP_ETIMEOUT, waits (bounded) for its own
// copies and products in flight, frees the tensor memory and returns.
#pragma once

#include "compose_append.cuh"
#include "decode_attn.cuh"

namespace yocopp {

struct PrefillParams {
    uint8_t* out;           // [total_q][hq][128] bf16
    const int32_t* pos;     // [batch] cache position of each sequence's first query row, or null (0)
    const int32_t* cu_q;    // [batch + 1] query-row offsets, or null (n_uniform rows per sequence)
    const int32_t* block_table;  // [batch][mbps] for a paged cache, or null (contiguous)
    int32_t n_uniform;
    int32_t batch, hq, hkv, capacity;
    int32_t block_size, mbps, num_blocks;  // paged cache only
    int32_t boxr;           // rows per K/V box: 128 (contiguous) or min(block_size, 128)
    int32_t q_tiles;        // ceil(max query rows per sequence / 128)
    int32_t heads_per_cta;  // 2 (group size even) or 1
    float qscale;           // softmax scale * log2(e)
    uint64_t wait_limit_ns;
    int32_t drop_k_tile;    // testing: K tile whose load CTA 0 never issues (-1: none)
    // fused composition (prefill_tc_kernel<true> only): raw rows of layer 1 and of
    // this layer, packed like q ([total_q][hkv][128] bf16), the weights, the cache
    // planes the composed rows go to, and the call generation and per-(sequence,
    // query tile) flags in the caller's workspace
    const uint8_t* k1;
    const uint8_t* v1;
    const uint8_t* ki;
    const uint8_t* vi;
    uint8_t* ck;
    uint8_t* cv;
    float ak1, ak2, av1, av2, lam;
    unsigned long long* ws_gen;  // [0] last finished call's generation, [1] call arrivals
    unsigned long long* flags;   // [batch][q_tiles]: generation of the call that composed the tile
};

struct PfShape {
    static constexpr int D = 128, TQ = 128, TK = 128;
    static constexpr int BOXB = 128 * 128;          // one [128 rows][128 B] swizzled box
    static constexpr int TILE_BYTES = 2 * BOXB;     // 128 rows x 128 channels, bf16
    static constexpr int KSLOTS = 2, VSLOTS = 2;
    static constexpr int Q_OFF = 0;                 // Q_a, Q_b
    static constexpr int K_OFF = 2 * TILE_BYTES;
    static constexpr int V_OFF = K_OFF + KSLOTS * TILE_BYTES;
    static constexpr int BAR_OFF = V_OFF + VSLOTS * TILE_BYTES;
    // q_full, k_full[2], k_empty[2], v_full[2], v_empty[2], s_full[2], p_full[2], o_done[2], drain,
    // o_last[2]
    static constexpr int NBAR = 18;
    static constexpr int SMEM = 1024 + BAR_OFF + NBAR * 8 + 16;
    static constexpr int THREADS = 320;
    static constexpr uint32_t IDESC_QK = umma_idesc_bf16(128, 128, false);
    static constexpr uint32_t IDESC_PV = umma_idesc_bf16(128, 128, true);
    static constexpr int TMEM_COLS = 512;           // S_a 0, S_b 128, O_a 256, O_b 384
    static constexpr float RESCALE_SLACK = 8.f;     // log2 of the largest P before a rescale
};
static_assert(PfShape::SMEM <= 232448 - 16, "prefill shared memory");

// 2^x on the FMA pipe for two arguments at once (fp32x2 arithmetic), for
// x <= 2^22 (x below -126 is taken as -126, whose result, at most 2^-125.5,
// is nothing next to the row's largest term 1; a causally masked key's -inf
// therefore gets a weight of at most 2^-125.5 here, where MUFU gives 0: the
// row sum is at least 2^-8, so such a key moves the output by at most 2^-117
// of its value row, which the fp32 sums cannot even represent, and its value
// row lies inside the window, so it is finite): x = j + f with j = round(x),
// f in [-1/2, 1/2] (Cody and Waite's range reduction, with the round done by
// adding 1.5 * 2^23), 2^f from a cubic fitted here to the relative error on
// [-1/2, 1/2] (max 7.5e-5, far below the 2^-8 rounding of the bf16 probabilities it
// feeds), and 2^j added to the exponent field.  The exponential unit does 16
// results per clock per SM, one tile's worth in the time the tensor cores take
// for it; moving a quarter of them here keeps it off the critical path.
__device__ __forceinline__ float2 exp2_poly2(float2 x) {
    x.x = fmaxf(x.x, -126.f);  // keeps the exponent field of the result >= 0
    x.y = fmaxf(x.y, -126.f);
    const float2 mg = make_float2(12582912.f, 12582912.f), nmg = make_float2(-12582912.f, -12582912.f);
    const float2 t = fadd2(x, mg);                                      // round(x) in the low mantissa bits
    const float2 f = ffma2(fadd2(t, nmg), make_float2(-1.f, -1.f), x);  // x - round(x), exact
    float2 p = ffma2(make_float2(0x1.c3f76p-5f, 0x1.c3f76p-5f), f, make_float2(0x1.f0de1ap-3f, 0x1.f0de1ap-3f));
    p = ffma2(p, f, make_float2(0x1.62f31ap-1f, 0x1.62f31ap-1f));
    p = ffma2(p, f, make_float2(0x1.fff692p-1f, 0x1.fff692p-1f));
    return make_float2(__int_as_float(__float_as_int(p.x) + (__float_as_int(t.x) << 23)),
                       __int_as_float(__float_as_int(p.y) + (__float_as_int(t.y) << 23)));
}

// max of three (sm_100 three-input max.f32; a NaN input is skipped as by fmaxf)
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// acc + the two bf16 of w (low half into .x), each widened exactly and added
// with one rounding (sm_100 mixed-precision add.f32.bf16): the sums that
// widening first and adding in fp32 give, without the widening instructions.
__device__ __forceinline__ float2 add_bf16x2(float2 acc, uint32_t w) {
    float2 r;
    asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %2;\n\t"
        "add.rn.f32.bf16 %0, lo, %3;\n\tadd.rn.f32.bf16 %1, hi, %4;\n\t}"
        : "=f"(r.x), "=f"(r.y)
        : "r"(w), "f"(acc.x), "f"(acc.y));
    return r;
}

// Pairs of keys whose two exponentials come from the cubic (one pair in four:
// a quarter of the exponentials on the FMA pipe, the rest on MUFU).
__device__ __forceinline__ constexpr bool poly_pair(int e) { return (e & 3) == 3; }

// Fused composition: compose query tile jt's rows of sequence b (every KV head)
// from the raw layer-1 and layer-i rows with the arithmetic of
// yocopp_compose_append (so the stored bits are the same) and write them to
// their cache positions p_b + jt * 128 + r.  The four input streams are
// contiguous here (the tile's (token, head) rows), so lane 0 of warp 0 stages
// them into shared memory with 1-D bulk copies, 64 rows (16 KB) of each
// stream per stage, three stages deep; warps 1..9 compose from shared memory
// and store the cache rows.  All threads of the CTA call it.
__device__ __forceinline__ void prefill_compose_tile(const PrefillParams& p, int b, int jt, int tid, uint8_t* smem) {
    using S = PfShape;
    constexpr int SROWS = 64, STAGES = 3, SBYTES = SROWS * 256;  // per stream and stage
    constexpr int NC = S::THREADS - 32;                           // composing threads
    static_assert(STAGES * 4 * SBYTES <= S::BAR_OFF, "composition stages fit below the barriers");
    int qrow0, nq;
    if (p.cu_q) {
        qrow0 = __ldg(p.cu_q + b);
        nq = __ldg(p.cu_q + b + 1) - qrow0;
    } else {
        qrow0 = b * p.n_uniform;
        nq = p.n_uniform;
    }
    const int p0 = p.pos ? __ldg(p.pos + b) : 0;
    // an invalid sequence is reported by its attention CTAs
    if (nq < 0 || p0 < 0 || int64_t(p0) + nq > p.capacity || nq > p.q_tiles * S::TQ) return;
    const int r0 = jt * S::TQ;
    const int n = min(S::TQ, nq - r0);
    if (n <= 0) return;
    const int rows = n * p.hkv;                                   // the tile's (token, head) rows
    const int nsb = (rows + SROWS - 1) / SROWS;
    const int64_t in0 = (int64_t(qrow0) + r0) * p.hkv * 256;      // byte offset of its first input row
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + S::BAR_OFF);
    uint64_t* empty = full + STAGES;
    const int warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], NC / 32);
        }
        fence_mbar_init();
    }
    __syncthreads();
    if (warp == 0) {
        if (lane == 0) {
            int issued = 0;
            for (int sb = 0; sb < nsb; ++sb) {
                const int st = sb % STAGES;
                if (!mbar_wait(&empty[st], ((sb / STAGES) & 1) ^ 1, p.wait_limit_ns)) {
                    record_status(YOCOPP_ETIMEOUT);
                    break;
                }
                const int r = sb * SROWS;
                const uint32_t bytes = uint32_t(min(SROWS, rows - r)) * 256u;
                mbar_arrive_expect_tx(&full[st], 4u * bytes);
                uint8_t* dst = smem + st * 4 * SBYTES;
                const int64_t off = in0 + int64_t(r) * 256;
                bulk_load(dst, p.k1 + off, bytes, &full[st]);
                bulk_load(dst + SBYTES, p.ki + off, bytes, &full[st]);
                bulk_load(dst + 2 * SBYTES, p.v1 + off, bytes, &full[st]);
                bulk_load(dst + 3 * SBYTES, p.vi + off, bytes, &full[st]);
                issued = sb + 1;
            }
            // the copies still in flight land before the CTA may exit
            for (int sb = issued > STAGES ? issued - STAGES : 0; sb < issued; ++sb)
                (void)mbar_wait(&full[sb % STAGES], (sb / STAGES) & 1, p.wait_limit_ns);
        }
        return;
    }
    const ComposeCoef ck = make_coef(p.ak1, p.ak2, p.lam);
    const ComposeCoef cv = make_coef(p.av1, p.av2, p.lam);
    const int ctid = tid - 32;
    for (int sb = 0; sb < nsb; ++sb) {
        const int st = sb % STAGES;
        if (!__all_sync(0xffffffffu, mbar_wait(&full[st], (sb / STAGES) & 1, p.wait_limit_ns))) {
            record_status(YOCOPP_ETIMEOUT);
            break;
        }
        const int r = sb * SROWS;
        const int nrow = min(SROWS, rows - r);
        const uint8_t* src = smem + st * 4 * SBYTES;
        for (int i = ctid; i < nrow * 16; i += NC) {
            const int lr = i >> 4, c = i & 15;
            const int row = r + lr;
            const int tok = row / p.hkv, h = row % p.hkv;
            const int position = p0 + r0 + tok;
            int64_t dst;
            if (p.block_table == nullptr) {
                dst = ((int64_t(b) * p.hkv + h) * p.capacity + position) * 256;
            } else {
                const int blk = __ldg(p.block_table + int64_t(b) * p.mbps + position / p.block_size);
                if (blk < 0 || blk >= p.num_blocks) {
                    record_status(YOCOPP_EDEVICE_CHECK);
                    continue;
                }
                dst = ((int64_t(blk) * p.hkv + h) * p.block_size + position % p.block_size) * 256;
            }
            const int so = lr * 256 + c * 16;
            const uint4 k1 = *reinterpret_cast<const uint4*>(src + so);
            const uint4 ki = *reinterpret_cast<const uint4*>(src + SBYTES + so);
            const uint4 v1 = *reinterpret_cast<const uint4*>(src + 2 * SBYTES + so);
            const uint4 vi = *reinterpret_cast<const uint4*>(src + 3 * SBYTES + so);
            st_global(p.ck + dst + c * 16, compose_chunk<__nv_bfloat16>(k1, ki, ck));
            st_global(p.cv + dst + c * 16, compose_chunk<__nv_bfloat16>(v1, vi, cv));
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[st]);
    }
}

// Wait (bounded) until the flag holds this call's generation.
__device__ __forceinline__ bool wait_flag(const unsigned long long* f, unsigned long long epoch, uint64_t limit_ns) {
    if (ld_acquire_gpu(f) == epoch) return true;
    const uint64_t t0 = globaltimer_ns();
    while (ld_acquire_gpu(f) != epoch) {
        if (globaltimer_ns() - t0 > limit_ns) return false;
        __nanosleep(128);
    }
    return true;
}

// FUSED: the grid also composes the rows it attends over.  Per sequence b there
// are q_tiles composition CTAs (one per 128-row query tile, every KV head) and
// the attention CTAs of the unfused kernel; the composition CTAs of sequence
// b + 1 are placed before the attention CTAs of sequence b, so they run one
// sequence ahead.  A composition CTA publishes its tile's flag (this call's
// generation, release) after its stores; an attention CTA's loaders wait
// (acquire, bounded) for the flags of every query tile whose rows a key tile
// holds before loading it.  Blocks are dispatched in index order, so every
// flag an attention CTA waits for belongs to a CTA that is already running or
// done, and no CTA waits on a later one.
template <bool FUSED>
__global__ void __launch_bounds__(PfShape::THREADS, 1)
prefill_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const PrefillParams p) {
    using S = PfShape;
    extern __shared__ uint8_t smem_raw[];
    __shared__ volatile int s_abort;
    __shared__ int s_cdone;

    griddep_wait();
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // CTA order: KV head planes one after another (sequence-major), and within a
    // plane the query tiles heaviest first, so that the CTAs resident at any
    // time stream the K/V tiles of one or two planes and find them in L2
    const int G = p.hq / p.hkv;
    const int units = G / p.heads_per_cta;                         // CTAs per (sequence, KV head, tile)
    const int per_plane = p.q_tiles * units;
    int bidx = int(blockIdx.x);                                    // index in the attention order
    unsigned long long epoch = 0;
    if constexpr (FUSED) {
        // every CTA reads the call's epoch (the last finished call's, + 1) and then arrives on
        // the call counter, off the critical path: the composition CTAs in one of their
        // composing threads, the attention CTAs in an idle lane of the loader warp
        const int per_attn = p.hkv * per_plane;
        int cb = -1, cjt = 0;
        if (bidx < p.q_tiles) {
            cb = 0;
            cjt = bidx;
        } else {
            const int i = bidx - p.q_tiles;
            const int sq = i / (p.q_tiles + per_attn), r = i % (p.q_tiles + per_attn);
            if (sq + 1 < p.batch && r < p.q_tiles) {
                cb = sq + 1;
                cjt = r;
            } else {
                bidx = sq * per_attn + (sq + 1 < p.batch ? r - p.q_tiles : r);
            }
        }
        if (cb >= 0) {
            __shared__ unsigned long long s_ep;
            if (tid == 32) {
                s_ep = __ldcg(p.ws_gen) + 1ull;
                arrive_call(p.ws_gen, s_ep, gridDim.x);
            }
            prefill_compose_tile(
                p, cb, cjt, tid,
                reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023)));
            fence_proxy_async_global();
            __threadfence();
            __syncthreads();
            if (tid == 0) st_release_gpu(p.flags + int64_t(cb) * p.q_tiles + cjt, s_ep);
            return;
        }
    }
    const int plane = bidx / per_plane;                            // b * hkv + g
    const int rem = bidx % per_plane;
    const int jt = p.q_tiles - 1 - rem / units;
    const int b = plane / p.hkv;
    const int g = plane % p.hkv;
    const int h0 = g * G + (rem % units) * p.heads_per_cta;
    const bool pair = p.heads_per_cta == 2;
    const int nsm = pair ? 8 : 4;                                  // softmax warps in use
    int qrow0, nq;
    if (p.cu_q) {
        qrow0 = __ldg(p.cu_q + b);
        nq = __ldg(p.cu_q + b + 1) - qrow0;
    } else {
        qrow0 = b * p.n_uniform;
        nq = p.n_uniform;
    }
    const int p0 = p.pos ? __ldg(p.pos + b) : 0;
    // FUSED: a CTA with nothing to do still arrives on the call counter
    auto leave = [&]() {
        if constexpr (FUSED) {
            if (tid == 0) arrive_call(p.ws_gen, __ldcg(p.ws_gen) + 1ull, gridDim.x);
        }
    };
    if (nq < 0) {
        if (tid == 0 && jt == 0 && g == 0 && rem % units == 0) record_status(YOCOPP_EDEVICE_CHECK);
        leave();
        return;
    }
    if (p0 < 0 || int64_t(p0) + nq > p.capacity || nq > p.q_tiles * S::TQ) {
        if (tid == 0 && jt == 0 && g == 0 && rem % units == 0) record_status(YOCOPP_ECAPACITY);
        leave();
        return;
    }
    if (jt * S::TQ >= nq) {
        leave();
        return;
    }
    const int kv_len = p0 + nq;
    const int jmax = min(jt * S::TQ + S::TQ - 1, nq - 1);
    const int ntk = (p0 + jmax) / S::TK + 1;        // key tiles 0 .. ntk-1 (causal)
    const int qpos_first = p0 + jt * S::TQ;          // smallest query position in the tile

    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(base + S::BAR_OFF);
    uint64_t* q_full = bars + 0;
    uint64_t* k_full = bars + 1;    // [2]
    uint64_t* k_empty = bars + 3;   // [2]
    uint64_t* v_full = bars + 5;    // [2]
    uint64_t* v_empty = bars + 7;   // [2]
    uint64_t* s_full = bars + 9;    // [head]
    uint64_t* p_full = bars + 11;   // [head]
    uint64_t* o_done = bars + 13;   // [head]
    uint64_t* drain = bars + 15;
    uint64_t* o_last = bars + 16;   // [head]: the CTA's last P V
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + S::BAR_OFF + S::NBAR * 8);

    if (tid == 0) {
        mbar_init(q_full, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&k_full[s], 1);
            mbar_init(&k_empty[s], 1);
            mbar_init(&v_full[s], 1);
            mbar_init(&v_empty[s], 1);
            mbar_init(&s_full[s], 1);
            mbar_init(&p_full[s], 4);
            mbar_init(&o_done[s], 1);
        }
        mbar_init(drain, 1);
        mbar_init(&o_last[0], 1);
        mbar_init(&o_last[1], 1);
        fence_mbar_init();
        s_abort = 0;
        s_cdone = 0;
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, S::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------------ producers
        int composed_upto = -1;  // FUSED: query tiles of this call seen composed
        if constexpr (FUSED) {
            // the query tiles first (they are inputs, not composed rows)
            if (lane == 0) {
                prefetch_tensormap(&tmQ);
                mbar_arrive_expect_tx(q_full, uint32_t((pair ? 2 : 1) * S::TILE_BYTES));
                for (int x = 0; x < (pair ? 2 : 1); ++x)
                    for (int bx = 0; bx < 2; ++bx)
                        tma_load_3d(base + S::Q_OFF + x * S::TILE_BYTES + bx * S::BOXB, &tmQ, q_full, bx * 64,
                                    h0 + x, qrow0 + jt * S::TQ);
            }
            if (lane == 2) epoch = __ldcg(p.ws_gen) + 1ull;
            epoch = __shfl_sync(0xffffffffu, epoch, 2);
            // one pass over every flag this CTA needs, 32 lanes x 4 loads in flight, then an
            // acquire fence per lane and a warp barrier: the tiles found ready (normally all:
            // their composition ran a sequence ahead) are not polled again
            const int last_pos = min(ntk * S::TK, kv_len) - 1;
            const int c_need = last_pos >= p0 ? (last_pos - p0) / S::TQ : -1;
            const unsigned long long* fl = p.flags + int64_t(b) * p.q_tiles;
            int first_missing = c_need + 1;
            for (int c0 = 0; c0 <= c_need; c0 += 128) {
                bool ready[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int c = c0 + 32 * k + lane;
                    ready[k] = c > c_need || ld_relaxed_gpu(fl + c) == epoch;
                }
                unsigned miss = 0;
#pragma unroll
                for (int k = 0; k < 4 && miss == 0; ++k) {
                    const unsigned m = __ballot_sync(0xffffffffu, !ready[k]);
                    if (m) {
                        miss = m;
                        first_missing = c0 + 32 * k + __ffs(m) - 1;
                    }
                }
                if (miss) break;
            }
            fence_acq_rel_gpu();
            __syncwarp();
            composed_upto = first_missing - 1;
            if (lane == 2) arrive_call(p.ws_gen, epoch, gridDim.x);
        }
        if (lane < 2) {
            const bool kl = lane == 0;   // lane 0: Q and the K ring; lane 1: the V ring
            const CUtensorMap* map = kl ? &tmK : &tmV;
            uint64_t* full = kl ? k_full : v_full;
            uint64_t* empty = kl ? k_empty : v_empty;
            uint8_t* ring = base + (kl ? S::K_OFF : S::V_OFF);
            int issued = 0;
            bool ok = true;
            prefetch_tensormap(map);
            if (kl && !FUSED) {
                prefetch_tensormap(&tmQ);
                mbar_arrive_expect_tx(q_full, uint32_t((pair ? 2 : 1) * S::TILE_BYTES));
                for (int x = 0; x < (pair ? 2 : 1); ++x)
                    for (int bx = 0; bx < 2; ++bx)
                        tma_load_3d(base + S::Q_OFF + x * S::TILE_BYTES + bx * S::BOXB, &tmQ, q_full, bx * 64,
                                    h0 + x, qrow0 + jt * S::TQ);
            }
            const int plane_row = (b * p.hkv + g) * p.capacity;
            const int nsb = S::TK / p.boxr;  // boxes of boxr rows per tile (one per cache block)
            if constexpr (FUSED) fence_proxy_async_global();
            for (int t = 0; t < ntk; ++t) {
                const int slot = t & 1;
                if (s_abort || !mbar_wait(&empty[slot], ((t >> 1) & 1) ^ 1, p.wait_limit_ns)) {
                    ok = false;
                    break;
                }
                if constexpr (FUSED) {
                    // this call's positions in the key tile come from query tiles .. c_hi
                    const int hi = min(t * S::TK + S::TK, kv_len) - 1;
                    if (hi >= p0) {
                        const int c_hi = (hi - p0) / S::TQ;
                        if (composed_upto < c_hi) {
                            while (ok && composed_upto < c_hi) {
                                ok = wait_flag(p.flags + int64_t(b) * p.q_tiles + composed_upto + 1, epoch,
                                               p.wait_limit_ns);
                                if (ok) ++composed_upto;
                            }
                            if (!ok) break;
                            fence_proxy_async_global();
                        }
                    }
                }
                if (kl && t == p.drop_k_tile && blockIdx.x == 0) continue;  // failure injection (tests)
                // the tile's rows: one 128-row box (contiguous), or one box per cache block;
                // blocks wholly past the sequence are not loaded (their K rows are masked and
                // their V rows zeroed before use)
                int rows[S::TK / 16];
                int nb = 0;
                for (int sb = 0; sb < nsb; ++sb) {
                    const int tok = t * S::TK + sb * p.boxr;
                    int row = -1;
                    if (p.block_table == nullptr) {
                        row = plane_row + tok;
                    } else if (tok < kv_len) {
                        const int blk = __ldg(p.block_table + int64_t(b) * p.mbps + tok / p.block_size);
                        if (blk < 0 || blk >= p.num_blocks)
                            record_status(YOCOPP_EDEVICE_CHECK);
                        else
                            row = (blk * p.hkv + g) * p.block_size + tok % p.block_size;
                    }
                    rows[sb] = row;
                    nb += row >= 0;
                }
                mbar_arrive_expect_tx(&full[slot], uint32_t(nb * p.boxr * 2 * 128));
                for (int sb = 0; sb < nsb; ++sb) {
                    if (rows[sb] < 0) continue;
                    for (int bx = 0; bx < 2; ++bx)
                        tma_load_2d(ring + slot * S::TILE_BYTES + bx * S::BOXB + sb * p.boxr * 128, map, &full[slot],
                                    bx * 64, rows[sb]);
                }
                issued = t + 1;
            }
            if (!ok) {
                record_status(YOCOPP_ETIMEOUT);
                s_abort = 1;
            }
            if (!ok || s_abort) {
                // let the copies this thread issued land before the CTA can exit
                if (kl) (void)mbar_wait(q_full, 0, p.wait_limit_ns);
                for (int t = issued > 2 ? issued - 2 : 0; t < issued; ++t)
                    (void)mbar_wait(&full[t & 1], (t >> 1) & 1, p.wait_limit_ns);
            }
        }
        return;
    }

    if (warp == 1) {
        // ------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t qaddr = smem_addr(base + S::Q_OFF);
            const uint32_t kaddr0 = smem_addr(base + S::K_OFF);
            const uint32_t vaddr0 = smem_addr(base + S::V_OFF);
            bool ok = mbar_wait(q_full, 0, p.wait_limit_ns);
            bool issued_any = false;
            auto qk = [&](int x, int t) {
                const uint32_t ka = kaddr0 + uint32_t((t & 1) * S::TILE_BYTES);
                const uint32_t qa = qaddr + uint32_t(x * S::TILE_BYTES);
#pragma unroll
                for (int kk = 0; kk < S::D / 16; ++kk) {
                    const uint32_t off = uint32_t((kk >> 2) * S::BOXB + (kk & 3) * 32);
                    umma_bf16(tmem + 128 * x, umma_desc_sw128(qa + off), umma_desc_sw128(ka + off), S::IDESC_QK,
                              kk > 0 ? 1u : 0u);
                }
                umma_commit(&s_full[x]);
                issued_any = true;
            };
            auto pv = [&](int x, int t) {
                const uint32_t va = vaddr0 + uint32_t((t & 1) * S::TILE_BYTES);
#pragma unroll
                for (int kk = 0; kk < S::TK / 16; ++kk)
                    umma_bf16_tmem_a(tmem + 256 + 128 * x, tmem + 128 * x + 8 * kk,
                                     umma_desc_sw128_mn(va + uint32_t(kk * 16 * 128), S::BOXB, 1024), S::IDESC_PV,
                                     (t > 0 || kk > 0) ? 1u : 0u);
                umma_commit(&o_done[x]);
                if (t == ntk - 1) umma_commit(&o_last[x]);
                issued_any = true;
            };
            if (ok) ok = !s_abort && mbar_wait(&k_full[0], 0, p.wait_limit_ns);
            if (ok) {
                tc_fence_after();
                qk(0, 0);
                if (pair) qk(1, 0);
                umma_commit(&k_empty[0]);
            }
            for (int t = 0; ok && t < ntk; ++t) {
                const bool more = t + 1 < ntk;
                // head a: P V of tile t, then S of tile t + 1
                if (s_abort || !mbar_wait(&p_full[0], t & 1, p.wait_limit_ns) ||
                    !mbar_wait(&v_full[t & 1], (t >> 1) & 1, p.wait_limit_ns)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                pv(0, t);
                if (more) {
                    if (!mbar_wait(&k_full[(t + 1) & 1], ((t + 1) >> 1) & 1, p.wait_limit_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    qk(0, t + 1);
                }
                if (pair) {
                    if (s_abort || !mbar_wait(&p_full[1], t & 1, p.wait_limit_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    pv(1, t);
                    if (more) qk(1, t + 1);
                }
                umma_commit(&v_empty[t & 1]);
                if (more) umma_commit(&k_empty[(t + 1) & 1]);
            }
            if (!ok) {
                record_status(YOCOPP_ETIMEOUT);
                s_abort = 1;
                if (issued_any) {  // every product issued finishes before the tensor memory is freed
                    umma_commit(drain);
                    (void)mbar_wait(drain, 0, p.wait_limit_ns);
                }
            }
            // the softmax warps finish reading O before the tensor memory is freed
            const uint64_t t0 = globaltimer_ns();
            while (atomicAdd(&s_cdone, 0) < nsm && globaltimer_ns() - t0 <= p.wait_limit_ns) __nanosleep(256);
        }
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, S::TMEM_COLS);
        return;
    }

    // ------------------------------------------------------------ softmax + epilogue
    const int x = (warp - 2) >> 2;                  // head of this warpgroup (0 = a, 1 = b)
    if (x == 1 && !pair) return;
    const int qd = warp & 3;
    const int r = 32 * qd + lane;                   // query row in the tile (TMEM lane)
    const int j = jt * S::TQ + r;                   // query row in the sequence
    const int qpos = p0 + j;                        // its cache position
    const uint32_t lanes = uint32_t(32 * qd) << 16;
    const uint32_t tS = tmem + 128 * x + lanes;     // this row's S (and P) in tensor memory
    const uint32_t tO = tmem + 256 + 128 * x + lanes;
    const float qscale = p.qscale;
    float m_ref = NEG_INF_F, l = 0.f;
    bool ok = true;
    for (int t = 0; t < ntk; ++t) {
        ok = __all_sync(0xffffffffu, !s_abort && mbar_wait(&s_full[x], t & 1, p.wait_limit_ns));
        if (!ok) break;
        tc_fence_after();
        const int key0 = t * S::TK;
        uint32_t u[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32_nowait(tS + uint32_t(c * 32), u[c]);
        tmem_wait_ld();
        if (key0 + S::TK - 1 > qpos_first) {  // tile reaches past some row's position: mask
#pragma unroll
            for (int c = 0; c < S::TK; ++c)
                if (key0 + c > qpos) u[c >> 5][c & 31] = __float_as_uint(NEG_INF_F);
        }
        float mx4[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) mx4[i] = __uint_as_float(u[0][i]);
#pragma unroll
        for (int c = 4; c < S::TK; c += 2)
            mx4[(c >> 1) & 3] = fmax3(mx4[(c >> 1) & 3], __uint_as_float(u[c >> 5][c & 31]),
                                      __uint_as_float(u[c >> 5][(c & 31) + 1]));
        const float mx = fmax3(fmaxf(mx4[0], mx4[1]), mx4[2], mx4[3]);
        const float m_new = fmaxf(m_ref, mx * qscale);
        const bool rescale = m_new > m_ref + S::RESCALE_SLACK;  // also when m_ref = -inf < m_new
        const float corr = rescale ? ex2_approx(m_ref - m_new) : 1.f;
        if (rescale) {
            l *= corr;
            m_ref = m_new;
        }
        // P = 2^(s - m) in bf16 into columns 0..63 of S (keys 2c, 2c + 1 in column c; S is
        // already in registers); one pair of keys in four from the polynomial, the rest from MUFU.
        // The row sum adds the bf16 values the product uses, so that the output is a convex
        // combination of V rows: its error is then sum_u w_u e_u (V_u - out) (e_u the relative
        // rounding of P_u), which vanishes where one key dominates.
        const float nmsub = m_ref == NEG_INF_F ? 0.f : -m_ref;
        const float2 qs2 = make_float2(qscale, qscale), nm2 = make_float2(nmsub, nmsub);
        float2 ls[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            uint32_t pw[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                const int k = 64 * c + 2 * e;
                const float2 xv = ffma2(make_float2(__uint_as_float(u[k >> 5][k & 31]),
                                                    __uint_as_float(u[k >> 5][(k & 31) + 1])), qs2, nm2);
                const float2 pe = poly_pair(e) ? exp2_poly2(xv) : make_float2(ex2_approx(xv.x), ex2_approx(xv.y));
                pw[e] = float2_to_bf16x2(pe.x, pe.y);
                ls[e & 1] = add_bf16x2(ls[e & 1], pw[e]);
            }
            tmem_st32u(tS + uint32_t(c * 32), pw);
        }
        l += (ls[0].x + ls[1].x) + (ls[0].y + ls[1].y);
        if (t > 0 && __any_sync(0xffffffffu, rescale)) {
            // bring O to the new reference (after P, so that S no longer occupies
            // registers): P V of the previous tile must have finished
            ok = __all_sync(0xffffffffu, mbar_wait(&o_done[x], (t - 1) & 1, p.wait_limit_ns));
            if (!ok) break;
            tc_fence_after();
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
                float o[32];
                tmem_ld32(tO + uint32_t(c * 32), o);
#pragma unroll
                for (int i = 0; i < 32; ++i) o[i] *= corr;
                tmem_st32(tO + uint32_t(c * 32), o);
            }
        }
        if (x == 0 && key0 + S::TK > kv_len) {
            // V rows past the sequence hold whatever the cache holds: zero them
            // (once the tile has landed, before either head's P V reads it) so
            // that the zero probabilities of those keys cannot meet a NaN
            ok = __all_sync(0xffffffffu, mbar_wait(&v_full[t & 1], (t >> 1) & 1, p.wait_limit_ns));
            if (!ok) break;
            if (key0 + r >= kv_len) {
                uint8_t* vrow = base + S::V_OFF + (t & 1) * S::TILE_BYTES + r * 128;
#pragma unroll
                for (int bx = 0; bx < 2; ++bx)
#pragma unroll
                    for (int cc = 0; cc < 8; ++cc)
                        *reinterpret_cast<uint4*>(vrow + bx * S::BOXB + cc * 16) = make_uint4(0u, 0u, 0u, 0u);
            }
            fence_proxy_async_smem();
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[x]);
    }
    // O is final once the CTA's last P V for this head has completed (a one-phase barrier,
    // so the wait cannot be confused by phase parity)
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&o_last[x], 0, p.wait_limit_ns));
    if (ok) {
        tc_fence_after();
        const float inv = l > 0.f ? 1.f / l : 0.f;
        const bool store = j < nq;
        uint8_t* orow = p.out + ((int64_t(qrow0) + j) * p.hq + h0 + x) * int64_t(S::D * 2);
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
            float o[32];
            tmem_ld32(tO + uint32_t(c * 32), o);
            if (store) {
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    uint4 v;
                    v.x = float2_to_bf16x2(o[q4 * 8 + 0] * inv, o[q4 * 8 + 1] * inv);
                    v.y = float2_to_bf16x2(o[q4 * 8 + 2] * inv, o[q4 * 8 + 3] * inv);
                    v.z = float2_to_bf16x2(o[q4 * 8 + 4] * inv, o[q4 * 8 + 5] * inv);
                    v.w = float2_to_bf16x2(o[q4 * 8 + 6] * inv, o[q4 * 8 + 7] * inv);
                    st_global(orow + (c * 32 + q4 * 8) * 2, v);
                }
            }
        }
    } else {
        record_status(YOCOPP_ETIMEOUT);
        s_abort = 1;
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) atomicAdd(&s_cdone, 1);
}

}  // namespace yocopp
