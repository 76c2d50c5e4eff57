// Gather-expand attention over selected micro-blocks (prefill and decode),
// and dense GQA decode as the special case "every block selected".
//
// "用125亿分之6的参数，打平3970亿的旗舰模型", section
// "稀疏注意力：给检索建索引，也得先学会省纸": the selected blocks are expanded
// back into their original tokens, which take part in the real attention.
// AITOP100 news page, section "二、架构 / 1. 注意力机制": full-precision
// attention over the selected blocks only.
//
// Work item = one query token (prefill) or one slice of one decode query's
// selection.  The item's blocks are gathered 4 tokens x all KV heads at a time
// (one contiguous 2 KiB run per block for K and for V at Hkv = 2, D = 128)
// with 16-byte cp.async into a shared-memory ring (2 stages in prefill, 3 in
// decode), XOR-swizzled for conflict-free ldmatrix.  With G = Hq / Hkv query
// heads per KV head, a token's work per KV head is M = G rows, too few for an
// MMA tile, so the MMA runs transposed: S^T = K_sel (16 keys) x Q^T (G <= 8 heads as N = 8).  The
// softmax runs per head column in registers (fp32, base-2 exponent), the
// probabilities are rounded to bf16 and moved into B-operand layout with
// movmatrix, and O^T = V_sel^T x P accumulates in fp32.  Warps of one KV head
// split the keys; their (max, sum, O) are merged through shared memory at the
// end of the item.  The kernel is bound by gather bandwidth (2 MiB per query
// token at budget 2048), not by the tensor pipe.
#include "qsa_common.cuh"
#include "qsa_launch.h"

namespace qsa {

namespace sat {

constexpr int WARPS = 4;
constexpr int THREADS = WARPS * 32;
constexpr float LOG2E = 1.4426950408889634f;
constexpr float LN2 = 0.6931471805599453f;

enum Mode { PREFILL = 0, SPLIT = 1 };

// Prefill: 2-stage ring, 3 CTAs per SM (12 warps: the gather is latency-bound
// and more resident warps beat a deeper ring).  Split decode: 3-stage ring,
// 2 CTAs per SM (few items per SM, a deeper ring per item pays).
template <int MODE>
struct Ring {
    static constexpr int STAGES = MODE == PREFILL ? 2 : 3;
    static constexpr int CTAS = MODE == PREFILL ? 3 : 2;
};

template <int D, int HKV, int STAGES>
struct Cfg {
    static constexpr int WPG = WARPS / HKV;           // warps per KV head
    static constexpr int KS = 16 * WPG;               // keys per stage
    static constexpr int NBS = KS / 4;                // blocks per stage
    static constexpr int ROW = HKV * D * 2;           // bytes of one key row (all heads)
    static constexpr int CHR = ROW / 16;              // 16-byte chunks per key row
    static constexpr int STAGE_K = KS * ROW;
    static constexpr int STAGE_BYTES = 2 * STAGE_K;   // K then V
    static constexpr int OFF_SEL = STAGES * STAGE_BYTES;
    static constexpr int MAX_ENT = 1024;
    static constexpr int BYTES = OFF_SEL + MAX_ENT * 4;
    // merge area (aliases the stage ring once it has drained)
    static constexpr int MERGE_BYTES = WARPS * (D * 8 + 16) * 4;
    static_assert(MERGE_BYTES <= STAGES * STAGE_BYTES, "merge area");
};

struct Args {
    const uint16_t *q;       // prefill [B,Tq,Hq,D]; split [B,Hq,D]
    const uint16_t *k;       // [B,Tk,Hkv,D]
    const uint16_t *v;
    const int32_t *sel;      // [rows, kb] or nullptr (dense: every block)
    const int64_t *q_pos0;   // prefill positions base, or nullptr
    const int32_t *seqlens;  // split mode: p = seqlens[b] - 1
    int B;
    int64_t Tq, Tk;
    int Hq;
    int kb;                  // entries per selection row
    int nsplit, chunk;       // split mode: entries per item
    float scale_log2;
    uint16_t *o;
    float *lse;
    float *part;             // split mode: [B, nsplit, Hq, D + 2]
    void *status;            // workspace (status word) or nullptr
    int64_t total_items;
};

template <int D, int G, int HKV, int MODE>
__global__ void __launch_bounds__(THREADS, Ring<MODE>::CTAS) sparse_attn_kernel(const Args a) {
    griddep_wait();  // the selection (and partial buffers) of the previous kernel
    constexpr int STAGES = Ring<MODE>::STAGES;
    using C = Cfg<D, HKV, STAGES>;
    constexpr int KSTEP = D / 16;
    extern __shared__ __align__(128) uint8_t smem[];
    int *s_blk = reinterpret_cast<int *>(smem + C::OFF_SEL);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int lr = lane >> 2, lc = lane & 3;
    const int g = warp / C::WPG, sub = warp % C::WPG;
    const int Hq = HKV * G;

    for (int64_t item = blockIdx.x; item < a.total_items; item += gridDim.x) {
        // ---- describe the item ------------------------------------------
        int64_t b, row, p;
        int e0, e1;
        const uint16_t *qrow;
        if (MODE == PREFILL) {
            row = item;
            b = row / a.Tq;
            const int64_t t = row - b * a.Tq;
            p = (a.q_pos0 ? a.q_pos0[b] : 0) + t;
            e0 = 0;
            e1 = a.kb;
            qrow = a.q + row * Hq * D;
        } else {
            b = item / a.nsplit;
            row = b;
            const int split = (int)(item - b * a.nsplit);
            p = (int64_t)a.seqlens[b] - 1;
            e0 = split * a.chunk;
            e1 = e0 + a.chunk;
            if (e1 > a.kb) e1 = a.kb;
            qrow = a.q + b * Hq * D;
        }
        if (p >= a.Tk || p < 0) {
            if (tid == 0) record_status(a.status, QSA_ERR_DEVICE);
            p = -1;  // empty token set
        }
        const int n_ent = e1 > e0 ? e1 - e0 : 0;
        const uint16_t *kb_ = a.k + b * a.Tk * HKV * D;
        const uint16_t *vb_ = a.v + b * a.Tk * HKV * D;
        for (int i = tid; i < n_ent; i += THREADS) {
            int j = a.sel ? a.sel[row * a.kb + e0 + i] : e0 + i;
            if (j < 0 || (int64_t)j * 4 > p) j = -1;
            s_blk[i] = j;
        }
        // Q^T fragments for this warp's KV head (heads g*G + n, n = lr < G)
        uint32_t bq[KSTEP][2];
#pragma unroll
        for (int ks = 0; ks < KSTEP; ++ks) {
            uint32_t v0 = 0, v1 = 0;
            if (lr < G) {
                const uint16_t *qh = qrow + (g * G + lr) * D + ks * 16 + 2 * lc;
                v0 = *reinterpret_cast<const uint32_t *>(qh);
                v1 = *reinterpret_cast<const uint32_t *>(qh + 8);
            }
            bq[ks][0] = v0;
            bq[ks][1] = v1;
        }
        __syncthreads();

        const int n_stage = (n_ent + C::NBS - 1) / C::NBS;
        // TPB threads copy one block: thread li of block bi takes chunks
        // li + TPB * k of the block's 4 key rows (block index read once)
        constexpr int TPB = THREADS / C::NBS;
        constexpr int MR = C::CHR / TPB;  // passes per key row
        static_assert(TPB * C::NBS == THREADS && MR * TPB == C::CHR, "copy split");
        const int bi = tid / TPB, li = tid % TPB;
        auto load_stage = [&](int s) {
            if (s < n_stage) {
                uint8_t *dk = smem + (s % STAGES) * C::STAGE_BYTES;
                uint8_t *dv = dk + C::STAGE_K;
                const int ent = s * C::NBS + bi;
                const int j = ent < n_ent ? s_blk[ent] : -1;
                const int64_t u0 = (int64_t)j * 4;
#pragma unroll
                for (int k = 0; k < 4 * MR; ++k) {
                    const int r = k / MR;                    // token of the block
                    const int ch = li + TPB * (k % MR);      // 16-byte chunk of its key row
                    const int kk = bi * 4 + r;
                    const bool ok = j >= 0 && u0 + r <= p;
                    const int64_t off = ok ? (u0 + r) * (HKV * D) + ch * 8 : 0;
                    // chunk ch of the key row = head ch / (D/8), dim chunk ch % (D/8)
                    const int hh = ch / (D / 8), dc = ch % (D / 8);
                    const int dst = kk * C::ROW + hh * D * 2 + ((dc ^ (kk & 7)) * 16);
                    cp_async16(smem_u32(dk + dst), kb_ + off, ok ? 16 : 0);
                    cp_async16(smem_u32(dv + dst), vb_ + off, ok ? 16 : 0);
                }
            }
            cp_async_commit();
        };
#pragma unroll
        for (int s = 0; s < STAGES - 1; ++s) load_stage(s);

        float m_run[2] = {-INFINITY, -INFINITY};
        float l_run[2] = {0.f, 0.f};
        float oacc[KSTEP][4];
#pragma unroll
        for (int mt = 0; mt < KSTEP; ++mt)
#pragma unroll
            for (int e = 0; e < 4; ++e) oacc[mt][e] = 0.f;

#pragma unroll 1
        for (int s = 0; s < n_stage; ++s) {
            cp_async_wait<STAGES - 2>();
            __syncthreads();
            load_stage(s + STAGES - 1);
            const uint8_t *sk = smem + (s % STAGES) * C::STAGE_BYTES + g * D * 2;
            const uint8_t *sv = sk + C::STAGE_K;
            // S^T = K (16 keys) x Q^T
            float sacc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int ks = 0; ks < KSTEP; ++ks) {
                const int mi = lane >> 3;
                const int kk = sub * 16 + (mi & 1) * 8 + (lane & 7);
                const int dc = ks * 2 + (mi >> 1);
                uint32_t a0, a1, a2, a3;
                ldmatrix_x4(smem_u32(sk + kk * C::ROW + ((dc ^ (kk & 7)) * 16)), a0, a1, a2, a3);
                mma_bf16_16816(sacc, a0, a1, a2, a3, bq[ks][0], bq[ks][1]);
            }
            // mask and scale: key rows lr and lr + 8 of this warp's m-tile
            float x[4];
#pragma unroll
            for (int hrow = 0; hrow < 2; ++hrow) {
                const int kk = sub * 16 + lr + hrow * 8;
                const int ent = s * C::NBS + (kk >> 2);
                const int j = ent < n_ent ? s_blk[ent] : -1;
                const bool ok = j >= 0 && (int64_t)j * 4 + (kk & 3) <= p;
                x[hrow * 2 + 0] = ok ? sacc[hrow * 2 + 0] * a.scale_log2 : -INFINITY;
                x[hrow * 2 + 1] = ok ? sacc[hrow * 2 + 1] * a.scale_log2 : -INFINITY;
            }
            float pr[4];
#pragma unroll
            for (int hc = 0; hc < 2; ++hc) {  // head column 2*lc + hc
                float mx = fmaxf(x[hc], x[2 + hc]);
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
                const float m_new = fmaxf(m_run[hc], mx);
                const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
                const float alpha = fast_exp2(m_run[hc] - m_use);
                pr[hc] = fast_exp2(x[hc] - m_use);
                pr[2 + hc] = fast_exp2(x[2 + hc] - m_use);
                l_run[hc] = l_run[hc] * alpha + pr[hc] + pr[2 + hc];
                m_run[hc] = m_new;
#pragma unroll
                for (int mt = 0; mt < KSTEP; ++mt) {
                    oacc[mt][hc] *= alpha;
                    oacc[mt][2 + hc] *= alpha;
                }
            }
            const uint32_t pb0 = movmatrix_trans(pack_bf16x2(pr[0], pr[1]));
            const uint32_t pb1 = movmatrix_trans(pack_bf16x2(pr[2], pr[3]));
            // O^T += V^T (dims x 16 keys) x P (16 keys x heads)
#pragma unroll
            for (int mt = 0; mt < KSTEP; ++mt) {
                const int mi = lane >> 3;
                const int kk = sub * 16 + (mi >> 1) * 8 + (lane & 7);
                const int dc = mt * 2 + (mi & 1);
                uint32_t a0, a1, a2, a3;
                ldmatrix_x4_trans(smem_u32(sv + kk * C::ROW + ((dc ^ (kk & 7)) * 16)), a0, a1,
                                  a2, a3);
                mma_bf16_16816(oacc[mt], a0, a1, a2, a3, pb0, pb1);
            }
        }
        cp_async_wait<0>();
        __syncthreads();

        // ---- merge the warps of each KV head -----------------------------
#pragma unroll
        for (int hc = 0; hc < 2; ++hc) {
            float l = l_run[hc];
            l += __shfl_xor_sync(0xffffffffu, l, 4);
            l += __shfl_xor_sync(0xffffffffu, l, 8);
            l += __shfl_xor_sync(0xffffffffu, l, 16);
            l_run[hc] = l;
        }
        float *mrg = reinterpret_cast<float *>(smem) + warp * (D * 8 + 16);
        if (lr == 0) {
            mrg[D * 8 + 2 * lc] = m_run[0];
            mrg[D * 8 + 2 * lc + 1] = m_run[1];
            mrg[D * 8 + 8 + 2 * lc] = l_run[0];
            mrg[D * 8 + 8 + 2 * lc + 1] = l_run[1];
        }
#pragma unroll
        for (int mt = 0; mt < KSTEP; ++mt) {
            mrg[(mt * 16 + lr) * 8 + 2 * lc] = oacc[mt][0];
            mrg[(mt * 16 + lr) * 8 + 2 * lc + 1] = oacc[mt][1];
            mrg[(mt * 16 + lr + 8) * 8 + 2 * lc] = oacc[mt][2];
            mrg[(mt * 16 + lr + 8) * 8 + 2 * lc + 1] = oacc[mt][3];
        }
        __syncthreads();
        for (int i = tid; i < HKV * G * D; i += THREADS) {
            const int d = i % D;
            const int n = (i / D) % G;
            const int gg = i / (D * G);
            float M = -INFINITY;
#pragma unroll
            for (int w = 0; w < C::WPG; ++w) {
                const float *m = reinterpret_cast<float *>(smem) + (gg * C::WPG + w) * (D * 8 + 16);
                M = fmaxf(M, m[D * 8 + n]);
            }
            const float Mu = (M == -INFINITY) ? 0.f : M;
            float L = 0.f, O = 0.f;
#pragma unroll
            for (int w = 0; w < C::WPG; ++w) {
                const float *m = reinterpret_cast<float *>(smem) + (gg * C::WPG + w) * (D * 8 + 16);
                const float f = fast_exp2(m[D * 8 + n] - Mu);
                L += m[D * 8 + 8 + n] * f;
                O += m[d * 8 + n] * f;
            }
            const int h = gg * G + n;
            if (MODE == PREFILL) {
                a.o[(row * Hq + h) * D + d] = to_bf16_bits(L > 0.f ? O / L : 0.f);
                if (a.lse && d == 0)
                    a.lse[row * Hq + h] = L > 0.f ? (M + __log2f(L)) * LN2 : -INFINITY;
            } else {
                float *pp = a.part + ((item * Hq) + h) * (D + 2);
                pp[d] = O;
                if (d == 0) {
                    pp[D] = M;
                    pp[D + 1] = L;
                }
            }
        }
        __syncthreads();
    }
}

// Merge split partials: one thread per (sequence, head, dim).
template <int D>
__global__ void __launch_bounds__(256) split_combine_kernel(const float *__restrict__ part,
                                                            int B, int Hq, int nsplit,
                                                            uint16_t *__restrict__ o,
                                                            float *__restrict__ lse) {
    griddep_wait();  // the split partials
    const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (i >= (int64_t)B * Hq * D) return;
    const int d = (int)(i % D);
    const int64_t bh = i / D;
    const int h = (int)(bh % Hq);
    const int64_t b = bh / Hq;
    float M = -INFINITY;
    for (int s = 0; s < nsplit; ++s)
        M = fmaxf(M, part[((b * nsplit + s) * Hq + h) * (D + 2) + D]);
    const float Mu = (M == -INFINITY) ? 0.f : M;
    float L = 0.f, O = 0.f;
    for (int s = 0; s < nsplit; ++s) {
        const float *pp = part + ((b * nsplit + s) * Hq + h) * (D + 2);
        const float f = fast_exp2(pp[D] - Mu);
        L += pp[D + 1] * f;
        O += pp[d] * f;
    }
    o[bh * D + d] = to_bf16_bits(L > 0.f ? O / L : 0.f);
    if (lse && d == 0) lse[bh] = L > 0.f ? (M + __log2f(L)) * LN2 : -INFINITY;
}

template <int D, int G, int HKV, int MODE>
static cudaError_t launch_sat(const Args &a, int grid, cudaStream_t s) {
    using C = Cfg<D, HKV, Ring<MODE>::STAGES>;
    auto kern = sparse_attn_kernel<D, G, HKV, MODE>;
    cudaError_t e = ensure_smem(reinterpret_cast<const void *>(kern), C::BYTES);
    if (e != cudaSuccess) return e;
    if (a.total_items == 0) return cudaSuccess;
    return launch_dependent(kern, dim3(grid), dim3(THREADS), (size_t)C::BYTES, s, a);
}

template <int MODE>
static cudaError_t dispatch(const Args &a, int D, int G, int Hkv, int grid, cudaStream_t s) {
#define QSA_SAT(D_, G_, H_) \
    if (D == D_ && G == G_ && Hkv == H_) return launch_sat<D_, G_, H_, MODE>(a, grid, s);
#define QSA_SAT_G(D_, H_) QSA_SAT(D_, 1, H_) QSA_SAT(D_, 2, H_) QSA_SAT(D_, 4, H_) QSA_SAT(D_, 8, H_)
    QSA_SAT_G(64, 1) QSA_SAT_G(64, 2) QSA_SAT_G(64, 4)
    QSA_SAT_G(128, 1) QSA_SAT_G(128, 2) QSA_SAT_G(128, 4)
#undef QSA_SAT_G
#undef QSA_SAT
    return cudaErrorInvalidValue;
}

}  // namespace sat

int sparse_attn_blocks_per_stage(int Hkv) { return 16 * (sat::WARPS / Hkv) / 4; }

cudaError_t launch_sparse_attn_prefill(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                                       const int32_t *sel, const int64_t *q_pos0, int B,
                                       int64_t Tq, int64_t Tk, int Hq, int Hkv, int D, int kb,
                                       float scale, uint16_t *o, float *lse, int num_sms,
                                       cudaStream_t s) {
    sat::Args a{};
    a.q = q; a.k = k; a.v = v; a.sel = sel; a.q_pos0 = q_pos0; a.seqlens = nullptr;
    a.B = B; a.Tq = Tq; a.Tk = Tk; a.Hq = Hq; a.kb = kb; a.nsplit = 1; a.chunk = kb;
    a.scale_log2 = scale * sat::LOG2E; a.o = o; a.lse = lse; a.part = nullptr;
    a.status = nullptr; a.total_items = (int64_t)B * Tq;
    int64_t grid = (int64_t)num_sms * sat::Ring<sat::PREFILL>::CTAS;
    if (grid > a.total_items) grid = a.total_items > 0 ? a.total_items : 1;
    return sat::dispatch<sat::PREFILL>(a, D, Hq / Hkv, Hkv, (int)grid, s);
}

// Split-K decode over a selection (sel != nullptr) or over all blocks
// 0..floor(p/4) (sel == nullptr, n_entries = L_max / 4 rounded up).
cudaError_t launch_split_decode(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                                const int32_t *seqlens, int64_t L_max, const int32_t *sel,
                                int n_entries, int nsplit, int B, int Hq, int Hkv, int D,
                                float scale, uint16_t *o, float *lse, float *part,
                                void *status, int num_sms, cudaStream_t s) {
    sat::Args a{};
    a.q = q; a.k = k; a.v = v; a.sel = sel; a.q_pos0 = nullptr; a.seqlens = seqlens;
    a.B = B; a.Tq = 1; a.Tk = L_max; a.Hq = Hq; a.kb = n_entries; a.nsplit = nsplit;
    a.chunk = (n_entries + nsplit - 1) / nsplit;
    a.scale_log2 = scale * sat::LOG2E; a.o = o; a.lse = lse; a.part = part;
    a.status = status; a.total_items = (int64_t)B * nsplit;
    const int64_t slots = (int64_t)num_sms * sat::Ring<sat::SPLIT>::CTAS;
    int64_t grid = a.total_items < slots ? a.total_items : slots;
    cudaError_t e = sat::dispatch<sat::SPLIT>(a, D, Hq / Hkv, Hkv, (int)(grid > 0 ? grid : 1), s);
    if (e != cudaSuccess) return e;
    const int64_t n = (int64_t)B * Hq * D;
    if (n == 0) return cudaSuccess;
    const dim3 cgrid((unsigned)((n + 255) / 256));
    if (D == 64)
        return launch_dependent(sat::split_combine_kernel<64>, cgrid, dim3(256), 0, s,
                                (const float *)part, B, Hq, nsplit, o, lse);
    return launch_dependent(sat::split_combine_kernel<128>, cgrid, dim3(256), 0, s,
                            (const float *)part, B, Hq, nsplit, o, lse);
}

}  // namespace qsa
