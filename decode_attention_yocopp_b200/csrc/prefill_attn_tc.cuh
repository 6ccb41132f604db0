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
// One CTA per (sequence, query head, 128-row query tile), heaviest query
// tiles first.  Tensor memory holds S (128 x 128 fp32, columns 0..127) and
// the output accumulator O (128 x 128 fp32, columns 128..255).  Per key tile:
//   S = Q K^T   eight tcgen05.mma (M = 128 queries, N = 128 keys, K = 16
//               channels each), Q and K K-major straight from their TMA tiles;
//   softmax     one thread per query row reads its S row, masks keys past
//               its position, and forms P = 2^(s - m) against a reference
//               maximum m that moves only when the row maximum exceeds it by
//               more than 8 (then O and the row sum are rescaled), so P <= 2^8
//               and the rescale is rare; P goes to shared memory as bf16 in
//               the 128-byte swizzled K-major layout the MMA reads;
//   O += P V    eight tcgen05.mma (M = 128, N = 128 channels, K = 16 keys)
//               with V read MN-major from its TMA tile.
// The next tile's S product is issued before this tile's P V so that the
// tensor cores work while the softmax threads do.
//
// Warps: 0 = TMA producer, 1 = MMA issuer and tensor-memory owner, 2..5 =
// softmax and epilogue (warp w reads TMEM lanes 32 (w mod 4) .. + 31).  Every
// wait is bounded; on a timeout the kernel records YOCOPP_ETIMEOUT, waits
// (bounded) for its own copies in flight, frees the tensor memory and returns.
#pragma once

#include "decode_attn.cuh"

namespace yocopp {

struct PrefillParams {
    uint8_t* out;           // [total_q][hq][128] bf16
    const int32_t* pos;     // [batch] cache position of each sequence's first query row, or null (0)
    const int32_t* cu_q;    // [batch + 1] query-row offsets, or null (n_uniform rows per sequence)
    int32_t n_uniform;
    int32_t batch, hq, hkv, capacity;
    int32_t q_tiles;        // ceil(max query rows per sequence / 128)
    float qscale;           // softmax scale * log2(e)
    uint64_t wait_limit_ns;
};

struct PfShape {
    static constexpr int D = 128, TQ = 128, TK = 128;
    static constexpr int BOXB = 128 * 128;          // one [128 rows][128 B] swizzled box
    static constexpr int TILE_BYTES = 2 * BOXB;     // 128 rows x 128 channels, bf16
    static constexpr int Q_OFF = 0;
    static constexpr int KV_OFF = TILE_BYTES;       // 2 stages x (K tile, V tile)
    static constexpr int P_OFF = KV_OFF + 4 * TILE_BYTES;
    static constexpr int BAR_OFF = P_OFF + TILE_BYTES;
    static constexpr int NBAR = 9;                  // q_full, kv_full[2], kv_empty[2], s_full, s_free, p_full, o_done
    static constexpr int SMEM = 1024 + BAR_OFF + NBAR * 8 + 16;
    static constexpr uint32_t IDESC_QK = umma_idesc_bf16(128, 128, false);
    static constexpr uint32_t IDESC_PV = umma_idesc_bf16(128, 128, true);
    static constexpr int TMEM_COLS = 256;
    static constexpr float RESCALE_SLACK = 8.f;     // log2 of the largest P before a rescale
};

__global__ void __launch_bounds__(192, 1)
prefill_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const PrefillParams p) {
    using S = PfShape;
    extern __shared__ uint8_t smem_raw[];
    __shared__ volatile int s_abort;
    __shared__ int s_cdone;

    griddep_wait();
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int per_tile = p.batch * p.hq;
    const int jt = p.q_tiles - 1 - int(blockIdx.x) / per_tile;  // heaviest (latest) query tiles first
    const int rem = int(blockIdx.x) % per_tile;
    const int b = rem / p.hq, h = rem % p.hq;
    const int g = h / (p.hq / p.hkv);
    int qrow0, nq;
    if (p.cu_q) {
        qrow0 = __ldg(p.cu_q + b);
        nq = __ldg(p.cu_q + b + 1) - qrow0;
    } else {
        qrow0 = b * p.n_uniform;
        nq = p.n_uniform;
    }
    const int p0 = p.pos ? __ldg(p.pos + b) : 0;
    if (nq < 0) {
        if (tid == 0 && jt == 0 && h == 0) record_status(YOCOPP_EDEVICE_CHECK);
        return;
    }
    if (p0 < 0 || int64_t(p0) + nq > p.capacity || nq > p.q_tiles * S::TQ) {
        if (tid == 0 && jt == 0 && h == 0) record_status(YOCOPP_ECAPACITY);
        return;
    }
    if (jt * S::TQ >= nq) return;
    const int kv_len = p0 + nq;
    const int jmax = min(jt * S::TQ + S::TQ - 1, nq - 1);
    const int ntk = (p0 + jmax) / S::TK + 1;        // key tiles 0 .. ntk-1 (causal)
    const int qpos_first = p0 + jt * S::TQ;          // smallest query position in the tile

    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* Qs = base + S::Q_OFF;
    uint8_t* Ps = base + S::P_OFF;
    uint64_t* bars = reinterpret_cast<uint64_t*>(base + S::BAR_OFF);
    uint64_t* q_full = bars + 0;
    uint64_t* kv_full = bars + 1;   // [2]
    uint64_t* kv_empty = bars + 3;  // [2]
    uint64_t* s_full = bars + 5;
    uint64_t* s_free = bars + 6;
    uint64_t* p_full = bars + 7;
    uint64_t* o_done = bars + 8;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + S::BAR_OFF + S::NBAR * 8);

    if (tid == 0) {
        mbar_init(q_full, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&kv_full[s], 1);
            mbar_init(&kv_empty[s], 1);
        }
        mbar_init(s_full, 1);
        mbar_init(s_free, 4);
        mbar_init(p_full, 4);
        mbar_init(o_done, 1);
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
    const uint32_t tS = tmem, tO = tmem + 128;

    if (warp == 0) {
        // ------------------------------------------------------------------ producer
        if (lane == 0) {
            int last_t[2] = {-1, -1};
            bool ok = true;
            prefetch_tensormap(&tmQ);
            prefetch_tensormap(&tmK);
            prefetch_tensormap(&tmV);
            mbar_arrive_expect_tx(q_full, uint32_t(S::TILE_BYTES));
            for (int bx = 0; bx < 2; ++bx)
                tma_load_3d(Qs + bx * S::BOXB, &tmQ, q_full, bx * 64, h, qrow0 + jt * S::TQ);
            const int plane_row = (b * p.hkv + g) * p.capacity;
            for (int t = 0; t < ntk; ++t) {
                const int st = t & 1;
                if (s_abort || !mbar_wait(&kv_empty[st], ((t >> 1) & 1) ^ 1, p.wait_limit_ns)) {
                    ok = false;
                    break;
                }
                uint8_t* ks = base + S::KV_OFF + st * 2 * S::TILE_BYTES;
                uint8_t* vs = ks + S::TILE_BYTES;
                mbar_arrive_expect_tx(&kv_full[st], uint32_t(2 * S::TILE_BYTES));
                const int row = plane_row + t * S::TK;
                for (int bx = 0; bx < 2; ++bx) {
                    tma_load_2d(ks + bx * S::BOXB, &tmK, &kv_full[st], bx * 64, row);
                    tma_load_2d(vs + bx * S::BOXB, &tmV, &kv_full[st], bx * 64, row);
                }
                last_t[st] = t;
            }
            if (!ok) {
                record_status(YOCOPP_ETIMEOUT);
                s_abort = 1;
            }
            if (!ok || s_abort) {
                // let the copies this thread issued land before the CTA can exit
                (void)mbar_wait(q_full, 0, p.wait_limit_ns);
                for (int st = 0; st < 2; ++st)
                    if (last_t[st] >= 0) (void)mbar_wait(&kv_full[st], (last_t[st] >> 1) & 1, p.wait_limit_ns);
            }
        }
        return;
    }

    if (warp == 1) {
        // ------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t qaddr = smem_addr(Qs);
            const uint32_t paddr = smem_addr(Ps);
            const uint32_t kvaddr = smem_addr(base + S::KV_OFF);
            bool ok = mbar_wait(q_full, 0, p.wait_limit_ns);
            int pv_issued = 0;
            auto issue_qk = [&](int t) -> bool {
                if (s_abort || !mbar_wait(&kv_full[t & 1], (t >> 1) & 1, p.wait_limit_ns) ||
                    !mbar_wait(s_free, (t & 1) ^ 1, p.wait_limit_ns))
                    return false;
                tc_fence_after();
                const uint32_t kaddr = kvaddr + uint32_t((t & 1) * 2 * S::TILE_BYTES);
#pragma unroll
                for (int kk = 0; kk < S::D / 16; ++kk) {
                    const uint32_t off = uint32_t((kk >> 2) * S::BOXB + (kk & 3) * 32);
                    umma_bf16(tS, umma_desc_sw128(qaddr + off), umma_desc_sw128(kaddr + off), S::IDESC_QK,
                              kk > 0 ? 1u : 0u);
                }
                umma_commit(s_full);
                return true;
            };
            if (ok) ok = issue_qk(0);
            for (int t = 0; ok && t < ntk; ++t) {
                if (t + 1 < ntk && !issue_qk(t + 1)) {
                    ok = false;
                    break;
                }
                if (s_abort || !mbar_wait(p_full, t & 1, p.wait_limit_ns)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t vaddr = kvaddr + uint32_t((t & 1) * 2 * S::TILE_BYTES + S::TILE_BYTES);
#pragma unroll
                for (int kk = 0; kk < S::TK / 16; ++kk) {
                    const uint32_t aoff = uint32_t((kk >> 2) * S::BOXB + (kk & 3) * 32);
                    umma_bf16(tO, umma_desc_sw128(paddr + aoff),
                              umma_desc_sw128_mn(vaddr + uint32_t(kk * 16 * 128), S::BOXB, 1024), S::IDESC_PV,
                              (t > 0 || kk > 0) ? 1u : 0u);
                }
                umma_commit(o_done);
                umma_commit(&kv_empty[t & 1]);
                pv_issued = t + 1;
            }
            if (!ok) {
                record_status(YOCOPP_ETIMEOUT);
                s_abort = 1;
            }
            // the softmax warps finish reading O before the tensor memory is freed
            const uint64_t t0 = globaltimer_ns();
            while (atomicAdd(&s_cdone, 0) < 4 && globaltimer_ns() - t0 <= p.wait_limit_ns) __nanosleep(256);
            if (!ok && pv_issued > 0) (void)mbar_wait(o_done, (pv_issued - 1) & 1, p.wait_limit_ns);
        }
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, S::TMEM_COLS);
        return;
    }

    // ------------------------------------------------------------ softmax + epilogue
    const int qd = warp & 3;
    const int r = 32 * qd + lane;                   // query row in the tile (TMEM lane)
    const int j = jt * S::TQ + r;                   // query row in the sequence
    const int qpos = p0 + j;                        // its cache position
    const uint32_t lanes = uint32_t(32 * qd) << 16;
    const float qscale = p.qscale;
    float m_ref = NEG_INF_F, l = 0.f;
    bool ok = true;
    for (int t = 0; t < ntk; ++t) {
        ok = __all_sync(0xffffffffu, !s_abort && mbar_wait(s_full, t & 1, p.wait_limit_ns));
        if (!ok) break;
        tc_fence_after();
        uint32_t u[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32_nowait(tS + lanes + uint32_t(c * 32), u[c]);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(s_free);

        const int key0 = t * S::TK;
        float mx = NEG_INF_F;
        if (key0 + S::TK - 1 > qpos_first) {  // tile reaches past some row's position: mask
#pragma unroll
            for (int c = 0; c < S::TK; ++c) {
                float v = __uint_as_float(u[c >> 5][c & 31]);
                v = (key0 + c <= qpos) ? v : NEG_INF_F;
                u[c >> 5][c & 31] = __float_as_uint(v);
                mx = fmaxf(mx, v);
            }
        } else {
#pragma unroll
            for (int c = 0; c < S::TK; ++c) mx = fmaxf(mx, __uint_as_float(u[c >> 5][c & 31]));
        }
        const float m_new = fmaxf(m_ref, mx * qscale);
        const bool rescale = m_new > m_ref + S::RESCALE_SLACK;  // also when m_ref = -inf < m_new
        const float corr = rescale ? ex2_approx(m_ref - m_new) : 1.f;
        if (rescale) {
            l *= corr;
            m_ref = m_new;
        }
        const float msub = m_ref == NEG_INF_F ? 0.f : m_ref;
        uint32_t pw[64];
        float lsum0 = 0.f, lsum1 = 0.f;
#pragma unroll
        for (int e = 0; e < 64; ++e) {
            const float a = ex2_approx(fmaf(__uint_as_float(u[(2 * e) >> 5][(2 * e) & 31]), qscale, -msub));
            const float c2 = ex2_approx(fmaf(__uint_as_float(u[(2 * e + 1) >> 5][(2 * e + 1) & 31]), qscale, -msub));
            lsum0 += a;
            lsum1 += c2;
            pw[e] = float2_to_bf16x2(a, c2);
        }
        l += lsum0 + lsum1;
        if (t > 0) {
            // P V of the previous tile has finished: O is final for it and P may be overwritten
            ok = __all_sync(0xffffffffu, mbar_wait(o_done, (t - 1) & 1, p.wait_limit_ns));
            if (!ok) break;
            tc_fence_after();
            if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll 1
                for (int c = 0; c < 4; ++c) {
                    float o[32];
                    tmem_ld32(tO + lanes + uint32_t(c * 32), o);
#pragma unroll
                    for (int i = 0; i < 32; ++i) o[i] *= corr;
                    tmem_st32(tO + lanes + uint32_t(c * 32), o);
                }
            }
        }
        uint8_t* prow = Ps + r * 128;
#pragma unroll
        for (int cc = 0; cc < 16; ++cc)
            *reinterpret_cast<uint4*>(prow + (cc >> 3) * S::BOXB + (((cc & 7) ^ (r & 7)) << 4)) =
                make_uint4(pw[4 * cc], pw[4 * cc + 1], pw[4 * cc + 2], pw[4 * cc + 3]);
        if (key0 + S::TK > kv_len && key0 + r >= kv_len) {
            // V rows past the sequence hold whatever the cache holds: zero them so
            // that the zero probabilities of those keys cannot meet a NaN
            uint8_t* vrow = base + S::KV_OFF + (t & 1) * 2 * S::TILE_BYTES + S::TILE_BYTES + r * 128;
#pragma unroll
            for (int bx = 0; bx < 2; ++bx)
#pragma unroll
                for (int cc = 0; cc < 8; ++cc)
                    *reinterpret_cast<uint4*>(vrow + bx * S::BOXB + cc * 16) = make_uint4(0u, 0u, 0u, 0u);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full);
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(o_done, (ntk - 1) & 1, p.wait_limit_ns));
    if (ok) {
        tc_fence_after();
        const float inv = l > 0.f ? 1.f / l : 0.f;
        const bool store = j < nq;
        uint8_t* orow = p.out + ((int64_t(qrow0) + j) * p.hq + h) * int64_t(S::D * 2);
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
            float o[32];
            tmem_ld32(tO + lanes + uint32_t(c * 32), o);
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
