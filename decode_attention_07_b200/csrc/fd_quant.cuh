// fd_quant.cuh -- the split kernel's consumer for an 8-bit key/value cache.
//
// Each cached element is a one-byte code, E4M3 (OCP 8-bit floating point:
// sign, 4 exponent bits with bias 7, 3 mantissa bits) or int8, with one
// scale per kv head: k = k_scale[h] * decode(code), v = v_scale[h] *
// decode(code). The "flash decoding论文" page lists INT8/INT4 quantisation
// among PaddleNLP's inference techniques; a cache of one byte per element
// halves the bytes the HBM-bound decode has to stream.
//
// The attention itself is unchanged (fd_split.cuh): per tile, logits, the
// online softmax and the rescaled accumulation of p * v, on tensor cores
// with mma.sync m16n8k16 for every group size (g = 1 included), because
// widening the codes already costs one instruction per two elements and the
// CUDA-core form would add a multiply-add per element on top.
//
//   * Codes are widened to f16 in registers, exactly: every E4M3 value and
//     every int8 value is an f16 value. f16 (not bf16) because the hardware
//     widens E4M3 pairs to f16 pairs in one instruction.
//   * The query is bf16; it enters the contraction as f16 after a per-column
//     power-of-two prescale that puts its largest element in [2^14, 2^15).
//     The prescale is exact, keeps every element inside f16's range, and
//     leaves only elements below 2^-25 of the column's largest rounded; the
//     logit multiplier of each column undoes it together with k_scale and
//     the softmax scale.
//   * Logits, S^T = K Q^T: ldmatrix of the 8-bit tile gives each thread four
//     consecutive codes of one token, which become the A fragment of one
//     16-element k-step once the query's B fragment is loaded in the same
//     order (q[4c .. 4c+3] per thread): the contraction index is only
//     permuted, identically on both sides.
//   * P V, O^T += V^T P^T: V must be transposed (tokens along k). ldmatrix
//     .trans of the 8-bit tile, read as 16-bit elements, hands each thread
//     two tokens x two head dims; one byte permute regroups them into token
//     pairs per head dim before widening. The accumulator rows then hold the
//     even head dims of a chunk (rows 0-7) and the odd ones (rows 8-15),
//     which the store at the end puts back in order.
//   * Softmax with a lazy reference maximum, after FlashDecoding++'s
//     asynchronous softmax with a unified max value (the "flash decoding论文"
//     page names the synchronised partial-softmax update as the problem it
//     removes): each column keeps a reference m and only a tile with a logit
//     above m + kLazy triggers the rescale of the running sum and the
//     accumulators; otherwise its p = 2^(x - m) is summed as is. The result
//     is the same softmax (m cancels in o / l and in the log-sum-exp); the
//     common tile skips the cross-lane max and the accumulator rescale.
//   * P enters as f16 high part + f16 remainder, scaled by 2^kPScale so that
//     small probabilities stay normal f16 numbers; the running sum carries
//     the same factor, so the normalised output is unchanged and only the
//     log-sum-exp is corrected (m - kPScale).
#pragma once

#include "fd_split.cuh"

namespace fd {

template <int D, int NT, bool kE4M3, int kTok = 16>
struct QuantConsumer {
    static constexpr int G = 8 * NT;        // columns held (padded)
    static constexpr int kElemBytes = 1;
    static constexpr int kWarpTokens = kTok;          // tokens of each tile per warp (16 or 32)
    static constexpr int MB = kTok / 16;              // 16-token blocks per warp
    static constexpr int KACC = MB == 1 ? 2 : 1;      // logit accumulators per block
    static constexpr bool kInterleaved = false;
    static constexpr int KC = D / 16;       // 16-byte chunks of a token = k-steps of S = m-tiles of O^T
    static constexpr int kRowBytes = D;
    // The reference max lags the running max by at most kLazy (base 2), so
    // p = 2^(x - m) <= 2^kLazy; P enters the P V product as p * 2^kPScale,
    // at most 2^15 (f16 tops out near 2^16) and a normal f16 down to p = 2^-21.
    static constexpr float kLazy = 8.f;
    static constexpr float kPScale = 7.f;

    uint32_t qf[NT][KC][2];                 // Q^T as the B operand (f16), per n-tile
    float m[NT][2], l[NT][2];               // reference max (base 2) / partial sum (x 2^kPScale), columns 2c, 2c+1
    float o[NT][KC][4];                     // O^T accumulators (x 2^kPScale, head dims even | odd per chunk)
    int shift[NT][2];                       // causal offset of columns 2c, 2c+1
    float colmul[NT][2];                    // logit multiplier (base 2) of columns 2c, 2c+1
    float kmul, vmul;                       // scale * log2(e) * k_scale[h], and v_scale[h]

    __device__ __forceinline__ void init(const SplitParams &p) {
        const int cc = (threadIdx.x & 31) & 3;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int col = nt * 8 + 2 * cc + e;
                shift[nt][e] = col < p.cols ? p.q_len - 1 - col / p.g : 0;
            }
    }

    __device__ __forceinline__ void set_row(const SplitParams &p, int h) {
        kmul = p.scale_log2e * __ldg(p.k_scale + h);
        vmul = __ldg(p.v_scale + h);
    }

    __device__ __forceinline__ void reset() {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            m[nt][0] = m[nt][1] = -INFINITY;
            l[nt][0] = l[nt][1] = 0.f;
#pragma unroll
            for (int c = 0; c < KC; ++c) o[nt][c][0] = o[nt][c][1] = o[nt][c][2] = o[nt][c][3] = 0.f;
        }
    }

    // 16-byte chunk `chunk` of tile row `row`, as TMA's swizzle placed it:
    // 128-byte rows (D = 128) use the 128-byte pattern, 64-byte rows the
    // 64-byte one (chunk bits xor address bits 7..8).
    static __device__ __forceinline__ int swz(int chunk, int row) {
        if constexpr (kRowBytes == 128)
            return chunk ^ (row & 7);
        else
            return chunk ^ ((row >> 1) & 3);
    }

    static __device__ __forceinline__ void widen(uint32_t w, uint32_t &lo, uint32_t &hi) {
        if constexpr (kE4M3)
            e4m3x4_to_f16(w, lo, hi);
        else
            int8x4_to_f16(w, lo, hi);
    }
    static __device__ __forceinline__ void widen_t(uint32_t w, uint32_t &lo, uint32_t &hi) {
        if constexpr (kE4M3)
            e4m3x4t_to_f16(w, lo, hi);
        else
            int8x4t_to_f16(w, lo, hi);
    }

    // Q^T fragments from the stage's bf16 copy of the row's columns ([cols][D]).
    __device__ __forceinline__ void load_q(const uint8_t *qs, int cols) {
        const int lane = threadIdx.x & 31;
        const int r0 = lane >> 2, cc = lane & 3;
        float cm[NT];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int col = nt * 8 + r0;
            const bool ok = col < cols;
            const uint2 *qrow = reinterpret_cast<const uint2 *>(qs + (ok ? col : 0) * D * 2);
            float qv[KC][4];
            float mx = 0.f;
#pragma unroll
            for (int c = 0; c < KC; ++c) {
                const uint2 w = qrow[4 * c + cc];   // q[16c + 4cc .. 16c + 4cc + 3]
                qv[c][0] = bf16lo_to_f32(w.x);
                qv[c][1] = bf16hi_to_f32(w.x);
                qv[c][2] = bf16lo_to_f32(w.y);
                qv[c][3] = bf16hi_to_f32(w.y);
#pragma unroll
                for (int e = 0; e < 4; ++e) mx = fmaxf(mx, fabsf(qv[c][e]));
            }
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));   // the 4 lanes of column r0
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
            const int ex = static_cast<int>((__float_as_uint(mx) >> 23) & 255u);
            const int j = ex == 0 ? 0 : min(141 - ex, 126);          // mx * 2^j in [2^14, 2^15)
            const float up = __uint_as_float(static_cast<uint32_t>(j + 127) << 23);
#pragma unroll
            for (int c = 0; c < KC; ++c) {
                qf[nt][c][0] = ok ? pack_f16x2(qv[c][0] * up, qv[c][1] * up) : 0u;
                qf[nt][c][1] = ok ? pack_f16x2(qv[c][2] * up, qv[c][3] * up) : 0u;
            }
            cm[nt] = kmul * __uint_as_float(static_cast<uint32_t>(127 - j) << 23);   // kmul * 2^-j
        }
        // the softmax needs the multipliers of columns 2cc, 2cc+1, held by lanes 4(2cc+e)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) colmul[nt][e] = __shfl_sync(0xffffffffu, cm[nt], 4 * (2 * cc + e));
    }

    static __device__ __forceinline__ uint32_t keep_tokens(uint32_t w, int t, int valid) {
        return w & ((t < valid ? 0x0000ffffu : 0u) | (t + 1 < valid ? 0xffff0000u : 0u));
    }

    // One tile: `slice` = this warp's slice of kWarpTokens tokens (MB blocks
    // of 16), `valid` = how many of those tokens are inside the row.
    __device__ __forceinline__ void tile(uint32_t k_smem, uint32_t v_smem, int slice, int valid, float) {
        const int lane = threadIdx.x & 31;
        const int mi = lane >> 3, rr = lane & 7;
        const int r0 = lane >> 2, cc = lane & 3;
        const int base = kWarpTokens * slice;

        // logits S^T = K Q^T per 16-token block; ldmatrix x4 over two chunks:
        // matrices (tokens 0-7 | 8-15) x (chunk 2pc | 2pc+1). One block keeps
        // two accumulators (even / odd chunks) for two independent mma
        // chains; two blocks already give two.
        float s[MB][KACC][NT][4];
#pragma unroll
        for (int mb = 0; mb < MB; ++mb)
#pragma unroll
            for (int a = 0; a < KACC; ++a)
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) s[mb][a][nt][e] = 0.f;
#pragma unroll
        for (int pc = 0; pc < KC / 2; ++pc) {
            const int chunk = 2 * pc + (mi >> 1);
#pragma unroll
            for (int mb = 0; mb < MB; ++mb) {
                const int lrow = base + 16 * mb + rr + 8 * (mi & 1);
                uint32_t a0, a1, a2, a3;
                ldsm_x4(k_smem + lrow * kRowBytes + (swz(chunk, lrow) << 4), a0, a1, a2, a3);
                uint32_t l0, h0, l1, h1, l2, h2, l3, h3;
                widen(a0, l0, h0);
                widen(a1, l1, h1);
                widen(a2, l2, h2);
                widen(a3, l3, h3);
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    mma_f16_16816(s[mb][0][nt], l0, l1, h0, h1, qf[nt][2 * pc][0], qf[nt][2 * pc][1]);
                    mma_f16_16816(s[mb][KACC - 1][nt], l2, l3, h2, h3, qf[nt][2 * pc + 1][0], qf[nt][2 * pc + 1][1]);
                }
            }
        }

        // Online softmax per column with a lazy reference maximum: m moves
        // (and the accumulators are rescaled) only when a logit of the tile
        // exceeds it by more than kLazy; otherwise p = 2^(x - m) directly.
        float x[MB][NT][4];
        bool grow = false;
#pragma unroll
        for (int mb = 0; mb < MB; ++mb)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    float acc = s[mb][0][nt][e];
                    if (KACC == 2) acc += s[mb][KACC - 1][nt][e];
                    x[mb][nt][e] = acc * colmul[nt][e & 1];
                }
                // token r of this block is inside column e's causal range when r < valid - 16 mb - shift
                const int va = valid - 16 * mb - shift[nt][0], vb = valid - 16 * mb - shift[nt][1];
                if (r0 >= va) x[mb][nt][0] = -INFINITY;
                if (r0 >= vb) x[mb][nt][1] = -INFINITY;
                if (r0 + 8 >= va) x[mb][nt][2] = -INFINITY;
                if (r0 + 8 >= vb) x[mb][nt][3] = -INFINITY;
                const float ta = m[nt][0] + kLazy, tb = m[nt][1] + kLazy;
                grow |= x[mb][nt][0] > ta || x[mb][nt][2] > ta || x[mb][nt][1] > tb || x[mb][nt][3] > tb;
            }
        if (__any_sync(0xffffffffu, grow)) {   // the fallback: a synchronised rescale
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                float ma = -INFINITY, mbx = -INFINITY;
#pragma unroll
                for (int mb = 0; mb < MB; ++mb) {
                    ma = fmaxf(ma, fmaxf(x[mb][nt][0], x[mb][nt][2]));
                    mbx = fmaxf(mbx, fmaxf(x[mb][nt][1], x[mb][nt][3]));
                }
#pragma unroll
                for (int sh = 4; sh < 32; sh <<= 1) {
                    ma = fmaxf(ma, __shfl_xor_sync(0xffffffffu, ma, sh));
                    mbx = fmaxf(mbx, __shfl_xor_sync(0xffffffffu, mbx, sh));
                }
                const float na = fmaxf(m[nt][0], ma), nb = fmaxf(m[nt][1], mbx);
                const float ua = na == -INFINITY ? 0.f : na, ub = nb == -INFINITY ? 0.f : nb;
                const float alpha_a = ex2(m[nt][0] - ua), alpha_b = ex2(m[nt][1] - ub);
                l[nt][0] *= alpha_a;
                l[nt][1] *= alpha_b;
                m[nt][0] = na;
                m[nt][1] = nb;
#pragma unroll
                for (int c = 0; c < KC; ++c) {
                    o[nt][c][0] *= alpha_a;
                    o[nt][c][1] *= alpha_b;
                    o[nt][c][2] *= alpha_a;
                    o[nt][c][3] *= alpha_b;
                }
            }
        }

        // P^T fragments per block (f16 high part + remainder, x 2^kPScale)
        uint32_t bh[MB][NT][2], bl[MB][NT][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const float ta = kPScale - (m[nt][0] == -INFINITY ? 0.f : m[nt][0]);
            const float tb = kPScale - (m[nt][1] == -INFINITY ? 0.f : m[nt][1]);
#pragma unroll
            for (int mb = 0; mb < MB; ++mb) {
                const float p0 = ex2(x[mb][nt][0] + ta), p2 = ex2(x[mb][nt][2] + ta);
                const float p1 = ex2(x[mb][nt][1] + tb), p3 = ex2(x[mb][nt][3] + tb);
                l[nt][0] += p0 + p2;
                l[nt][1] += p1 + p3;
                const uint32_t h01 = pack_f16x2(p0, p1), h23 = pack_f16x2(p2, p3);
                const uint32_t l01 = pack_f16x2(p0 - f16lo_to_f32(h01), p1 - f16hi_to_f32(h01));
                const uint32_t l23 = pack_f16x2(p2 - f16lo_to_f32(h23), p3 - f16hi_to_f32(h23));
                bh[mb][nt][0] = movmatrix_trans(h01);
                bh[mb][nt][1] = movmatrix_trans(h23);
                bl[mb][nt][0] = movmatrix_trans(l01);
                bl[mb][nt][1] = movmatrix_trans(l23);
            }
        }

        // O^T += V^T P^T, one 16-element chunk of head dims per m-tile, one
        // 16-token k-step per block. ldmatrix.trans of the 8-bit tile read as
        // 16-bit elements gives each thread tokens (2cc, 2cc+1) x head dims
        // (2r0, 2r0+1) of a chunk; the widening regroups them into token pairs
        // at head dims 2r0 (accumulator row r0) and 2r0 + 1 (row r0 + 8).
#pragma unroll
        for (int pc = 0; pc < KC / 2; ++pc) {
            const int chunk = 2 * pc + (mi >> 1);
#pragma unroll
            for (int mb = 0; mb < MB; ++mb) {
                const int lrow = base + 16 * mb + rr + 8 * (mi & 1);
                const int vmb = valid - 16 * mb;
                uint32_t a[4];
                ldsm_x4_trans(v_smem + lrow * kRowBytes + (swz(chunk, lrow) << 4), a[0], a[1], a[2], a[3]);
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    // tokens 0..7 (x) and 8..15 (y) of the block, chunk 2pc + half
                    uint32_t A0, A1, A2, A3;
                    widen_t(a[2 * half], A0, A1);
                    widen_t(a[2 * half + 1], A2, A3);
                    if (vmb < 16) {   // rows past the end may hold anything (NaN codes): zero them
                        A0 = keep_tokens(A0, 2 * cc, vmb);
                        A1 = keep_tokens(A1, 2 * cc, vmb);
                        A2 = keep_tokens(A2, 8 + 2 * cc, vmb);
                        A3 = keep_tokens(A3, 8 + 2 * cc, vmb);
                    }
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        mma_f16_16816(o[nt][2 * pc + half], A0, A1, A2, A3, bh[mb][nt][0], bh[mb][nt][1]);
                        mma_f16_16816(o[nt][2 * pc + half], A0, A1, A2, A3, bl[mb][nt][0], bl[mb][nt][1]);
                    }
                }
            }
        }
    }

    // This warp's (o, m, l) into a merge buffer slot: o[G][D] with the head
    // dims back in order and the value scale applied, then m[G] (base 2,
    // without the 2^kPScale factor), l[G].
    __device__ __forceinline__ void to_smem(float *wb) {
        constexpr int S = merge_head_stride<D>();
        const int lane = threadIdx.x & 31;
        const int r0 = lane >> 2, cc = lane & 3;
        const int dlo = 2 * r0;   // head dim of accumulator row r0 within its chunk (row r0 + 8: dlo + 1)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
            for (int e = 0; e < 2; ++e)
#pragma unroll
                for (int sh = 4; sh < 32; sh <<= 1) l[nt][e] += __shfl_xor_sync(0xffffffffu, l[nt][e], sh);
            const int ha = nt * 8 + 2 * cc, hb = ha + 1;
            // dims d0 and d0 + 1 of one head as one 8-byte store; with the padded
            // head stride the 16 lanes of each half warp fill all 32 banks
#pragma unroll
            for (int c = 0; c < KC; ++c) {
                const int d0 = 16 * c + dlo;
                *reinterpret_cast<float2 *>(wb + ha * S + d0) = make_float2(o[nt][c][0] * vmul, o[nt][c][2] * vmul);
                *reinterpret_cast<float2 *>(wb + hb * S + d0) = make_float2(o[nt][c][1] * vmul, o[nt][c][3] * vmul);
            }
            if (r0 == 0) {
                wb[G * S + ha] = m[nt][0] == -INFINITY ? -INFINITY : m[nt][0] - kPScale;
                wb[G * S + hb] = m[nt][1] == -INFINITY ? -INFINITY : m[nt][1] - kPScale;
                wb[G * S + G + ha] = l[nt][0];
                wb[G * S + G + hb] = l[nt][1];
            }
        }
    }
};

}  // namespace fd
