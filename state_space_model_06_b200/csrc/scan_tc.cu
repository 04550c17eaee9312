// scan_tc.cu -- chunked prefill of the Mamba-3 recurrence on tcgen05 tensor cores.
//
// Math (Mamba-3 paper summary, "Technical Approach"):
//   The exponential-trapezoidal complex recurrence (Propositions 1 and 4) is run in
//   chunks of Q tokens: inside a chunk the parallel masked form of "Parallel
//   representation under SSD" (Y = (L o C B^T) X with L = L_decay . L_band), across
//   chunks the recurrence on the N x P state.  The rotation is absorbed into B and C
//   (the RoPE trick, Proposition 3/4) with angles accumulated from the chunk start.
//
//   For chunk c with tokens t0..t1, chunk-relative log-decay cum_t = sum_{k=t0..t} dt_k A_k,
//   chunk-relative angle psi_t = sum_{k=t0..t} dt_k theta_k, rotated B~_u = R(-psi_u) B_u,
//   C~_t = R(-psi_t) C_t and the carried state g (original frame, with the next token's
//   trapezoid term already folded in):
//     Y_t   = sum_{u<=t} e^{cum_t-cum_u} (u<t ? w_u : gamma_u) (C~_t . B~_u) X_u
//             + e^{cum_t} C~_t^T g  +  D X_t
//     g'    = R(psi_t1) [ e^{cum_t1} g + sum_u e^{cum_t1-cum_u} w_u B~_u X_u^T ]
//     w_u   = gamma_u + (1 - lam_{u+1}) dt_{u+1}     (the beta term of token u+1)
//     g_0   = h0 + (1 - lam_0) dt_0 B_prev x_prev^T   (carried previous token)
//   At the end of the call w_{T-1} = gamma_{T-1}, so the last g' is exactly h_{T-1}.
//   MIMO: rows are (token, rank) pairs; L is shared by the R x R blocks.
//
// Kernel: one CTA per (batch, head), persistent over the chunks of the sequence.
//   warp 0       TMA producer (dt/A/lam per chunk, raw B, C, theta sub-chunks; zero fill past T)
//   warp 1       tcgen05.mma issuer:  S = C~ B~^T,  dS = B~^T (w-scaled X),
//                Y_inter = C~ g,  Y_intra = (S o L) X      (fp32 accumulators in TMEM)
//   warps 2-5    epilogue: mask S -> bf16 (S o L); y = Y_intra + e^{cum} Y_inter over the x tile
//   warps 6-13   rotation: cumulative angles, sincos, rotate B and C into swizzled bf16 MMA
//                operands, w-scaled X
//   warp 14      coefficients: log2-decay prefix (warp scan), gamma, w, mask exponent offsets
//   warp 15      x tiles in, y tiles out (TMA)
//   warps 16-19  state: g in TMEM (fp32), g <- e^{cum_end} g + dS, bf16 copy for Y_inter,
//                h_T rotated back to the original frame at the end of the call
// Every wait is bounded; a timeout raises a CTA-wide abort and records
// M3_ERR_TIMEOUT in the workspace status word.
#include <cuda.h>

#include <cstring>

#include "m3_internal.h"
#include "sm100.cuh"

namespace m3 {

using namespace sm100;

namespace {

constexpr int kP = 64;               // head dimension handled by this kernel
constexpr int kThreads = 640;       // 20 warps: TMA, MMA, 4 epilogue, 8 rotation, coefficients,
                                     // TMA x / y, 4 state
constexpr int kRotWarps = 8;
constexpr int kCoefSlots = 4;       // ring of per-chunk coefficient slots
constexpr int kTmemCols = 512;
constexpr float kLog2e = 1.4426950408889634f;

enum Bar {
    RAW_FULL0, RAW_FULL1, RAW_EMPTY0, RAW_EMPTY1,
    DT_FULL0, DT_FULL1, DT_EMPTY0, DT_EMPTY1,
    X_FULL0, X_FULL1, X_FULL2,
    COEF_FULL0, COEF_FULL1, COEF_FULL2, COEF_FULL3, COEF_EMPTY0, COEF_EMPTY1, COEF_EMPTY2,
    COEF_EMPTY3, CUM_READY0, CUM_READY1, CUM_READY2, CUM_READY3, RS0, RS1,
    OPS_FULL0, OPS_FULL1, OPS_EMPTY0, OPS_EMPTY1, S_FULL, S_EMPTY, SL_FULL, DS_FULL, DS_EMPTY,
    G_FULL, G_EMPTY, Y_FULL0, Y_FULL1, Y_EMPTY0, Y_EMPTY1, Y_STAGED0, Y_STAGED1, Y_STAGED2, DRAIN,
    NEVER, XR_FULL, NUM_BARS
};

// arrival count of each barrier: 1 for TMA expect_tx / tcgen05.commit / single-thread or
// single-warp arrivals, 4 for one elected lane per warp of a four-warp group, 5 for the
// coefficient slots (x warp + the four state warps), 8 for the rotation warps, 9 where the
// coefficient warp joins them.  Every barrier that a role waits on can complete its next
// phase only after that role has passed the current one (each y stage has its own
// Y_STAGED barrier for this reason), so no waiter can miss a phase.
__device__ __forceinline__ uint32_t bar_count(int i) {
    switch (i) {
        case DT_EMPTY0: case DT_EMPTY1: case COEF_FULL0: case COEF_FULL1: case COEF_FULL2:
        case COEF_FULL3:
            return kRotWarps + 1;
        case RAW_EMPTY0: case RAW_EMPTY1: case RS0: case RS1: case OPS_FULL0: case OPS_FULL1:
            return kRotWarps;
        case COEF_EMPTY0: case COEF_EMPTY1: case COEF_EMPTY2: case COEF_EMPTY3:
            return 5;
        case S_EMPTY: case SL_FULL: case DS_EMPTY: case G_FULL:
        case Y_EMPTY0: case Y_EMPTY1: case Y_STAGED0: case Y_STAGED1: case Y_STAGED2:
            return 4;
        default:
            return 1;
    }
}

template <int NST, int Q, int R, bool GT>
struct Cfg {
    static constexpr int L = Q * R;                 // rows of the intra-chunk tiles
    static constexpr int PAIRS = NST / 2;
    static constexpr int PB = PAIRS / 32;           // rotation warps along the pairs (1 or 2)
    static constexpr int TSPLIT = kRotWarps / PB;   // rotation warps along the tokens (8 or 4)
    static_assert(L == 64 || L == 128, "rows per chunk must be 64 or 128");
    static_assert(NST == 64 || NST == 128, "dstate must be 64 or 128");

    // bytes of the buffers
    static constexpr int X_BYTES = L * 128;
    static constexpr int DT_BOX = (Q + 1) * 16;                 // 4 heads x (Q+1) tokens, fp32
    static constexpr int DT_BYTES = (DT_BOX + 127) / 128 * 128;  // 128-byte aligned tiles
    static constexpr int CT_BYTES = (NST / 64) * L * 128;
    static constexpr int XW_BYTES = L * 128;
    static constexpr int SLOT_BYTES = 2 * CT_BYTES + XW_BYTES;  // C~, B~, Xw of one chunk
    static constexpr int SL_BYTES = (L / 64) * L * 128;
    static constexpr int G_BYTES = NST * 128;
    static constexpr int COEF_FLOATS = 4 * Q + PAIRS + 4;
    static constexpr int base_bytes() {
        return SL_BYTES + G_BYTES + 2 * 3 * DT_BYTES + kCoefSlots * COEF_FLOATS * 4 +
               2 * TSPLIT * PAIRS * 4 + NUM_BARS * 8 + 64;
    }
    // a raw stage: B, C (bf16), theta (fp32) and the BCNorm scales of B and C (fp32, [2][R][rt],
    // padded to 128 bytes; fetched only with BCNorm)
    static constexpr int sc_bytes(int rt) { return (2 * R * rt * 4 + 127) / 128 * 128; }
    static constexpr int raw_bytes(int rt) {
        return rt * R * NST * 2 * 2 + rt * PAIRS * 4 + sc_bytes(rt);
    }
    static constexpr int kSmemLimit = 232448 - 1024;            // minus base alignment slack
    // with the output gate, every x / y stage has a z tile beside it
    static constexpr int XZ_BYTES = (GT ? 2 : 1) * X_BYTES;
    // (operand slots, x stages, raw sub-chunk tokens): prefer two operand slots, then the
    // largest raw sub-chunk, then three x stages.  Every raw sub-chunk costs the rotation warps
    // an angle-sum exchange and a hand-off, so the sub-chunk size comes before the x stages:
    // the rank-4 MIMO tile (N 64, 32 tokens) went from 8-token sub-chunks with 3 x stages to
    // 16-token sub-chunks with 2, 1.84 -> 1.64 ms per 1.5B-scale MIMO call on B200.
    static constexpr int pick() {
        for (int ops = 2; ops >= 1; --ops)
            for (int rt = (Q < 32 ? Q : 32); rt >= TSPLIT; rt /= 2)
                for (int xst = 3; xst >= 2; --xst)
                    if (Q % rt == 0 && rt % TSPLIT == 0 &&
                        base_bytes() + ops * SLOT_BYTES + xst * XZ_BYTES + 2 * raw_bytes(rt) <=
                            kSmemLimit)
                        return ops * 10000 + xst * 1000 + rt;
        return 0;
    }
    static_assert(pick() != 0, "shared memory budget exceeded");
    static constexpr int OPS = pick() / 10000;                  // operand slots
    static constexpr int XST = (pick() / 1000) % 10;            // x / y staging stages
    static_assert(XST >= 2 && XST <= 3, "one Y_STAGED barrier per x / y stage");
    static constexpr int RT = pick() % 1000;                    // tokens per raw sub-chunk
    static constexpr int NSUB = Q / RT;
    static constexpr int TPT = RT / TSPLIT;                     // tokens per rotation thread
    static constexpr int BRAW_BYTES = RT * R * NST * 2;
    static constexpr int TH_BYTES = RT * PAIRS * 4;
    static constexpr int SC_OFF = 2 * BRAW_BYTES + TH_BYTES;    // BCNorm scales in a raw stage
    static constexpr int SC_BOX = 2 * R * RT * 4;               // bytes the scale copy delivers
    static constexpr int RAW_BYTES = SC_OFF + sc_bytes(RT);
    static_assert(SC_OFF % 128 == 0 && RAW_BYTES % 128 == 0, "TMA destinations must be aligned");

    // shared memory offsets (SW128 tiles first, 1024-byte aligned)
    static constexpr int OFF_X = 0;                                   // [XST] x / y staging
    static constexpr int OFF_Z = OFF_X + XST * X_BYTES;               // [XST] z (gate only)
    static constexpr int OFF_OPS = OFF_X + XST * XZ_BYTES;            // [OPS] C~, B~, Xw
    static constexpr int OFF_SL = OFF_OPS + OPS * SLOT_BYTES;         // S o L
    static constexpr int OFF_G = OFF_SL + SL_BYTES;                   // g (bf16)
    static constexpr int OFF_RAW = OFF_G + G_BYTES;                   // [2] B, C, theta
    static constexpr int OFF_DT = OFF_RAW + 2 * RAW_BYTES;            // [2] dt, A, lam
    static constexpr int OFF_COEF = OFF_DT + 2 * 3 * DT_BYTES;        // [kCoefSlots] coefficients
    static constexpr int OFF_RSUM = OFF_COEF + kCoefSlots * COEF_FLOATS * 4;  // [2][TSPLIT][PAIRS]
                                                                      // range angle sums
    static constexpr int OFF_BAR = (OFF_RSUM + 2 * TSPLIT * PAIRS * 4 + 7) / 8 * 8;
    static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;           // tmem base, abort flag
    // + alignment slack; at least 120 KB so that only one CTA fits on an SM (each CTA
    // allocates all 512 TMEM columns)
    static constexpr int SMEM_USED = OFF_MISC + 16 + 1024;
    static constexpr int SMEM = SMEM_USED > 122880 ? SMEM_USED : 122880;
    static_assert(SMEM <= 232448, "shared memory budget exceeded");
    static_assert(OFF_RAW % 128 == 0 && OFF_DT % 128 == 0, "TMA destinations must be aligned");
    __device__ static uint8_t* ct(uint8_t* sm, int slot) { return sm + OFF_OPS + slot * SLOT_BYTES; }
    __device__ static uint8_t* bt(uint8_t* sm, int slot) {
        return sm + OFF_OPS + slot * SLOT_BYTES + CT_BYTES;
    }
    __device__ static uint8_t* xw(uint8_t* sm, int slot) {
        return sm + OFF_OPS + slot * SLOT_BYTES + 2 * CT_BYTES;
    }

    // TMEM columns
    // TMEM columns: S, dS, and two buffers of (Y_intra, Y_inter)
    static constexpr uint32_t TM_S = 0, TM_DS = 128, TM_G = 448;   // G: the fp32 carried state
    __device__ static uint32_t tm_ya(int yb) { return 192u + 128u * yb; }
    __device__ static uint32_t tm_yi(int yb) { return 256u + 128u * yb; }

    // instruction descriptors
    static constexpr uint32_t ID_S = idesc_bf16(L, L, false, false);
    static constexpr uint32_t ID_DS = idesc_bf16(NST, kP, true, true);
    static constexpr uint32_t ID_Y = idesc_bf16(L, kP, false, true);
};

struct TcParams {
    CUtensorMap tm_x, tm_y, tm_z, tm_B, tm_C, tm_th, tm_dt, tm_A, tm_lam, tm_sc;
    CUtensorMap tm_xr, tm_zr;   // one value per head channel (MIMO lightweight expansion)
    ScanArgs a;
    int nch_total;      // chunks of the call
    int S;              // segments per (batch, head); 1: the call is one segment
    float* seg;         // segment records (S > 1), see seg_rec_floats
    unsigned long long limit_ns;
};

// Segment records, fp32, one per (segment s, batch * head bh) at index s * batch * H + bh:
//   M    [N][P]  the segment's final state when it starts from no state (segment pass)
//   G0   [N][P]  the segment's initial state g_0: h0 plus the first token's beta term for
//                segment 0; the beta term alone from the segment pass and the entry state
//                added by the chain step for the others
//   dec          the segment's total decay, e^{sum of its log-decays}
//   psi  [N/2]   the angles of the segment's final frame (segment-relative)
__host__ __device__ constexpr size_t seg_rec_floats(int N, int P) {
    return 2 * (size_t)N * P + 4 + N / 2;
}
__host__ __device__ constexpr size_t seg_off_g0(int N, int P) { return (size_t)N * P; }
__host__ __device__ constexpr size_t seg_off_dec(int N, int P) { return 2 * (size_t)N * P; }
__host__ __device__ constexpr size_t seg_off_psi(int N, int P) { return 2 * (size_t)N * P + 4; }

// One CTA's share of the call: (batch b, head h, segment s).  The call's chunks are split
// into S contiguous runs ("Parallel representation under SSD": the carried state is an
// affine function of the state entering the run, so runs compose).  The segment pass
// (MAP) runs segments 0 .. S-2 from no entry state (segment S-1 only prepares its g_0);
// the output pass runs every segment from its prepared g_0.
struct Unit {
    int b, h, g, s;
    size_t bh;
    int nch;              // chunks this launch runs for the unit
    long long t0, tend;   // the segment's first token and its end (exclusive)
    bool last;            // the segment holds the call's last token
};
template <int Q, bool MAP>
__device__ __forceinline__ Unit unit_of(const TcParams& p) {
    const ScanArgs& a = p.a;
    const int BH = a.batch * a.H;
    Unit u;
    u.s = (int)(blockIdx.x / BH);
    u.bh = blockIdx.x % BH;
    u.b = (int)(u.bh / a.H);
    u.h = (int)(u.bh % a.H);
    u.g = u.h / (a.H / a.G);
    const int c0 = (int)((long long)u.s * p.nch_total / p.S);
    const int c1 = (int)((long long)(u.s + 1) * p.nch_total / p.S);
    u.last = u.s == p.S - 1;
    u.nch = (MAP && u.last) ? 0 : c1 - c0;
    u.t0 = (long long)c0 * Q;
    u.tend = u.last ? a.T : (long long)c1 * Q;
    return u;
}

// coefficient slot layout (floats): cum2[Q] | gam[Q] | w[Q] | ew[Q] | psi_end[N/2] | cum2_end
//   cum2: chunk-relative log2-decay prefix; ew_u = log2(w_u) - cum2_u (mask exponent offset);
//   psi_end: call-relative angle of each pair at the chunk end (reduced mod 2 pi)
template <int NST, int Q, int R>
struct Coef {
    float* base;
    __device__ float* cum2() const { return base; }
    __device__ float* gam() const { return base + Q; }
    __device__ float* w() const { return base + 2 * Q; }
    __device__ float* ew() const { return base + 3 * Q; }
    __device__ float* psi_end() const { return base + 4 * Q; }
    __device__ float* cum2_end() const { return base + 4 * Q + NST / 2; }
};

__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// SiLU(z) = z * sigmoid(z) = z * (1/2 + tanh(z/2) / 2) for the output gate ("Technical
// Approach", output gating): one hardware tanh (relative error ~2^-11, below the bf16
// rounding of y that this kernel writes) instead of an exponential and a division.
__device__ __forceinline__ float tanh_approx(float x) {
    float y;
    asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float silu_fast(float z) {
    return z * fmaf(0.5f, tanh_approx(0.5f * z), 0.5f);
}

// A wait taken by all 32 lanes of a warp together: the outcome is made warp-uniform so
// that no lane reaches a .sync.aligned tcgen05 instruction without the others.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, const Abort& ab) {
    const bool r = mbar_wait(bar, parity, ab);
    return __all_sync(0xffffffffu, r);
}

// K-major SW128 operand, K step k (16 elements): atoms of 64 K-elements are `rows`*128 B apart.
__device__ __forceinline__ uint64_t desc_k(uint32_t base, int k, int rows) {
    return sdesc_sw128(base + (uint32_t)(k >> 2) * rows * 128u + (uint32_t)(k & 3) * 32u, 16u,
                       1024u);
}
// MN-major SW128 operand, K step k (16 rows of 128 B); MN atoms are `lbo` bytes apart.
__device__ __forceinline__ uint64_t desc_mn(uint32_t base, int k, uint32_t lbo) {
    return sdesc_sw128(base + (uint32_t)k * 2048u, lbo, 1024u);
}

// ---------------------------------------------------------------------------------
template <int NST, int Q, int R, bool GT, bool BC, bool MAP>
__device__ void producer(const TcParams& p, const Unit& u, uint8_t* sm, uint64_t* bar,
                         const Abort& ab);

// ---------------------------------------------------------------------------------
// ---------------------------------------------------------------------------------
template <int NST, int Q, int R, bool GT, bool MAP>
__device__ void mma_issuer(const TcParams& p, const Unit& u, uint8_t* sm, uint64_t* bar,
                           uint32_t tmem, const Abort& ab) {
    using C = Cfg<NST, Q, R, GT>;
    const uint32_t s_sl = smem_u32(sm + C::OFF_SL), s_g = smem_u32(sm + C::OFF_G);
    // failure-path test hook: wait on a barrier nothing completes (bounded, then abort)
    if ((p.a.flags & M3_FLAG_TEST_STALL) && !mbar_wait(&bar[NEVER], 0, ab)) return;
    for (int c = 0; c < u.nch; ++c) {
        const uint32_t ph = c & 1;
        const int yb = c & 1;
        const int slot = c % C::OPS;
        const uint32_t s_ct = smem_u32(C::ct(sm, slot)), s_bt = smem_u32(C::bt(sm, slot));
        const uint32_t s_xw = smem_u32(C::xw(sm, slot));
        if (!mbar_wait(&bar[OPS_FULL0 + slot], (c / C::OPS) & 1, ab)) return;
        if constexpr (MAP) {
            // segment pass: dS only.  Once the operands are published the rotation warps
            // no longer read x(c) or the chunk's coefficients: release the stage for the x
            // warp (in place of the four epilogue warps of the output pass).
            const int xs = c % C::XST;
#pragma unroll
            for (int i = 0; i < 4; ++i) mbar_arrive(&bar[Y_STAGED0 + xs]);
            if (!mbar_wait(&bar[DS_EMPTY], ph ^ 1, ab)) return;
            tc_fence_after();
#pragma unroll
            for (int k = 0; k < C::L / 16; ++k)
                mma_bf16(tmem + C::TM_DS, desc_mn(s_bt, k, C::L * 128u), desc_mn(s_xw, k, 1024u),
                         C::ID_DS, k > 0);
            mma_commit(&bar[DS_FULL]);
            mma_commit(&bar[OPS_EMPTY0 + slot]);
            continue;
        }
        tc_fence_after();
        // S = C~ B~^T   (M = L tokens*ranks, N = L, K = NST)
        if (!mbar_wait(&bar[S_EMPTY], ph ^ 1, ab)) return;
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < NST / 16; ++k)
            mma_bf16(tmem + C::TM_S, desc_k(s_ct, k, C::L), desc_k(s_bt, k, C::L), C::ID_S, k > 0);
        mma_commit(&bar[S_FULL]);
        // dS = B~^T Xw  (M = NST, N = P, K = L)
        if (!mbar_wait(&bar[DS_EMPTY], ph ^ 1, ab)) return;
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < C::L / 16; ++k)
            mma_bf16(tmem + C::TM_DS, desc_mn(s_bt, k, C::L * 128u), desc_mn(s_xw, k, 1024u),
                     C::ID_DS, k > 0);
        mma_commit(&bar[DS_FULL]);
        // Y_inter = C~ g  (M = L, N = P, K = NST)
        if (!mbar_wait(&bar[G_FULL], ph, ab)) return;
        if (!mbar_wait(&bar[Y_EMPTY0 + yb], ((c >> 1) & 1) ^ 1, ab)) return;
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < NST / 16; ++k)
            mma_bf16(tmem + C::tm_yi(yb), desc_k(s_ct, k, C::L), desc_mn(s_g, k, 1024u), C::ID_Y,
                     k > 0);
        mma_commit(&bar[G_EMPTY]);
        mma_commit(&bar[OPS_EMPTY0 + slot]);
        // Y_intra = (S o L) X  (M = L, N = P, K = L)
        if (!mbar_wait(&bar[SL_FULL], ph, ab)) return;
        const int xs = c % C::XST;
        if (!mbar_wait(&bar[X_FULL0 + xs], (c / C::XST) & 1, ab)) return;
        tc_fence_after();
        const uint32_t s_x = smem_u32(sm + C::OFF_X + xs * C::X_BYTES);
#pragma unroll
        for (int k = 0; k < C::L / 16; ++k)
            mma_bf16(tmem + C::tm_ya(yb), desc_k(s_sl, k, C::L), desc_mn(s_x, k, 1024u), C::ID_Y,
                     k > 0);
        mma_commit(&bar[Y_FULL0 + yb]);
    }
}

// ---------------------------------------------------------------------------------
// Rotation warps: B~ and C~ operands.  Rotation warp rw handles state pair
// 32*(rw % PB) + lane and tokens [ts*TPT, (ts+1)*TPT) of every raw sub-chunk, with
// ts = rw / PB.  The starting angle of a thread's token range is the running angle plus
// the angle sums of the earlier ranges, exchanged through shared memory once per
// sub-chunk (bounded mbarrier hand-off).
template <int NST, int Q, int R, bool GT, bool BC, bool MAP>
__device__ void rotation(const TcParams& p, const Unit& u, uint8_t* sm, uint64_t* bar,
                         const Abort& ab) {
    using C = Cfg<NST, Q, R, GT>;
    constexpr int TPT = C::TPT, PAIRS = C::PAIRS, TSPLIT = C::TSPLIT;
    const ScanArgs& a = p.a;
    const int tid = threadIdx.x - 192;          // 0..255
    const int rw = tid >> 5, lane = tid & 31;
    const int ts = rw / C::PB;
    const int pair = (rw % C::PB) * 32 + lane;   // this thread's state pair
    const int hq = u.h & 3;                      // column of this head in the 4-head dt tile
    const bool angle = (a.flags & M3_FLAG_THETA_IS_ANGLE) != 0;
    const int atom = (2 * pair) >> 6, col = (2 * pair) & 63;
    float* rsum = reinterpret_cast<float*>(sm + C::OFF_RSUM);
    int raw_it = 0;
    // BC map ("Technical Approach", BCNorm and BC biases): B and C of this thread's pair
    // channels become v * s + bias, s the column's BCNorm scale (1 when off), bias the head's
    constexpr bool bc = BC;
    const int hh = u.h;
    float bb0 = 0.f, bb1 = 0.f, cb0 = 0.f, cb1 = 0.f;
    if (a.B_bias) { bb0 = a.B_bias[hh * NST + 2 * pair]; bb1 = a.B_bias[hh * NST + 2 * pair + 1]; }
    if (a.C_bias) { cb0 = a.C_bias[hh * NST + 2 * pair]; cb1 = a.C_bias[hh * NST + 2 * pair + 1]; }
    const bool has_sc = a.bc_scale != nullptr;       // BCNorm scales come with the raw stage
    // segment-relative angle of this thread's pair (the RoPE frame of Proposition 4 starts at
    // the first token of the segment), reduced mod 2 pi at chunk boundaries
    float psi_acc = 0.f;
    for (int c = 0; c < u.nch; ++c) {
        const int st = c & 1, slot = c % C::OPS;
        const uint32_t ph2 = (c >> 1) & 1;
        if (!warp_wait(&bar[DT_FULL0 + st], ph2, ab)) return;
        const float* dtt = reinterpret_cast<const float*>(sm + C::OFF_DT + st * 3 * C::DT_BYTES);
        uint8_t* ct = C::ct(sm, slot);
        uint8_t* bt = C::bt(sm, slot);
        if (!warp_wait(&bar[OPS_EMPTY0 + slot], ((c / C::OPS) & 1) ^ 1, ab)) return;
        for (int s = 0; s < C::NSUB; ++s, ++raw_it) {
            const int rs = raw_it & 1;
            if (!warp_wait(&bar[RAW_FULL0 + rs], (raw_it >> 1) & 1, ab)) return;
            const uint8_t* raw = sm + C::OFF_RAW + rs * C::RAW_BYTES;
            const uint32_t* braw = reinterpret_cast<const uint32_t*>(raw);
            const uint32_t* craw = reinterpret_cast<const uint32_t*>(raw + C::BRAW_BYTES);
            const float* th = reinterpret_cast<const float*>(raw + 2 * C::BRAW_BYTES);
            const int tb = s * C::RT;           // first token of the sub-chunk (chunk-relative)
            const int j0 = ts * TPT;
            // angle increments of the own tokens and their sum
            // (running sums over the own tokens, one FMA each)
            float ph[TPT], own = 0.f;
#pragma unroll
            for (int jj = 0; jj < TPT; ++jj) {
                const int j = j0 + jj;
                const float d = angle ? 1.f : dtt[(tb + j) * 4 + hq];
                own = fmaf(d, th[j * PAIRS + pair], own);
                ph[jj] = own;
            }
            // publish the range sum; load the own tokens' raw B, C meanwhile
            float* rb = rsum + (rs * TSPLIT) * PAIRS;
            rb[ts * PAIRS + pair] = own;
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar[RS0 + rs]);
            uint32_t bv[TPT][R], cv[TPT][R];
#pragma unroll
            for (int jj = 0; jj < TPT; ++jj)
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    const int e = (((j0 + jj) * R + r) * NST) / 2 + pair;
                    bv[jj][r] = braw[e];
                    cv[jj][r] = MAP ? 0u : craw[e];   // the segment pass needs no C~
                }
            // BCNorm scales of the own tokens, [2][R][RT] in the raw stage (0 past the end
            // of the call, where B and C are zero-filled and the rows are masked out)
            float sb[TPT][R], sc[TPT][R];
            if constexpr (bc) {
                const float* scs = reinterpret_cast<const float*>(raw + C::SC_OFF);
#pragma unroll
                for (int jj = 0; jj < TPT; ++jj)
#pragma unroll
                    for (int r = 0; r < R; ++r) {
                        sb[jj][r] = has_sc ? scs[r * C::RT + j0 + jj] : 1.f;
                        sc[jj][r] = has_sc ? scs[(R + r) * C::RT + j0 + jj] : 1.f;
                    }
            }
            if (!warp_wait(&bar[RS0 + rs], (raw_it >> 1) & 1, ab)) return;
            float pre = 0.f, tot = 0.f;
#pragma unroll
            for (int qq = 0; qq < TSPLIT; ++qq) {
                const float v = rb[qq * PAIRS + pair];
                tot += v;
                pre += (qq < ts) ? v : 0.f;
            }
            const float psi0 = psi_acc + pre;
            float cn[TPT], sn[TPT];
#pragma unroll
            for (int jj = 0; jj < TPT; ++jj)   // |psi| < pi + one chunk of angle increments
                __sincosf(psi0 + ph[jj], &sn[jj], &cn[jj]);
            // operand rows (tb + j0 + jj) * R + r; when the first of them is a multiple of 8
            // the SW128 chunk of every row is a compile-time xor of this thread's chunk
            const int row0 = (tb + j0) * R;
            uint8_t* const cbase = ct + (uint32_t)atom * C::L * 128u + (uint32_t)(col & 7) * 2u;
            const uint32_t cx = (uint32_t)((col >> 3) & 7);
            auto store = [&](int jj, int r, uint32_t bo, uint32_t co) {
                const int k = jj * R + r;
                uint32_t off;
                if constexpr ((TPT * R) % 8 == 0 && (C::RT * R) % 8 == 0)
                    off = (uint32_t)(row0 + k) * 128u + ((cx ^ (uint32_t)(k & 7)) << 4);
                else
                    off = (uint32_t)(row0 + k) * 128u + ((cx ^ (uint32_t)((row0 + k) & 7)) << 4);
                *reinterpret_cast<uint32_t*>(cbase + C::CT_BYTES + off) = bo;
                if constexpr (!MAP) *reinterpret_cast<uint32_t*>(cbase + off) = co;
            };
            // R(-psi) [v0; v1] = [cos v0 + sin v1; -sin v0 + cos v1]
            if constexpr (!bc) {
                // on the packed bf16 pair itself: (v0, v0) (cos, -sin) + (v1, v1) (sin, cos)
#pragma unroll
                for (int jj = 0; jj < TPT; ++jj) {
                    const __nv_bfloat162 k0 = __floats2bfloat162_rn(cn[jj], -sn[jj]);
                    const __nv_bfloat162 k1 = __floats2bfloat162_rn(sn[jj], cn[jj]);
#pragma unroll
                    for (int r = 0; r < R; ++r) {
                        const uint32_t ub = bv[jj][r], uc = cv[jj][r];
                        const __nv_bfloat162 vb = *reinterpret_cast<const __nv_bfloat162*>(&ub);
                        const __nv_bfloat162 vc = *reinterpret_cast<const __nv_bfloat162*>(&uc);
                        const __nv_bfloat162 nb =
                            __hfma2(__high2bfloat162(vb), k1, __hmul2(__low2bfloat162(vb), k0));
                        const __nv_bfloat162 nc =
                            __hfma2(__high2bfloat162(vc), k1, __hmul2(__low2bfloat162(vc), k0));
                        store(jj, r, *reinterpret_cast<const uint32_t*>(&nb),
                              *reinterpret_cast<const uint32_t*>(&nc));
                    }
                }
            } else {
            // two tokens per packed fp32x2 operation (their cos and sin form the packed operands)
#pragma unroll
            for (int jj = 0; jj + 1 < TPT; jj += 2) {
                const float2 c2 = make_float2(cn[jj], cn[jj + 1]);
                const float2 s2 = make_float2(sn[jj], sn[jj + 1]);
                const float2 m2 = make_float2(-sn[jj], -sn[jj + 1]);
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    const uint32_t ba = bv[jj][r], bb = bv[jj + 1][r];
                    const uint32_t ca = cv[jj][r], cb = cv[jj + 1][r];
                    float2 b0 = make_float2(bf16lo(ba), bf16lo(bb));
                    float2 b1 = make_float2(bf16hi(ba), bf16hi(bb));
                    float2 c0 = make_float2(bf16lo(ca), bf16lo(cb));
                    float2 c1 = make_float2(bf16hi(ca), bf16hi(cb));
                    if constexpr (bc) {
                        const float2 sb2 = make_float2(sb[jj][r], sb[jj + 1][r]);
                        const float2 sc2 = make_float2(sc[jj][r], sc[jj + 1][r]);
                        b0 = __ffma2_rn(b0, sb2, make_float2(bb0, bb0));
                        b1 = __ffma2_rn(b1, sb2, make_float2(bb1, bb1));
                        c0 = __ffma2_rn(c0, sc2, make_float2(cb0, cb0));
                        c1 = __ffma2_rn(c1, sc2, make_float2(cb1, cb1));
                    }
                    const float2 nb0 = __ffma2_rn(c2, b0, __fmul2_rn(s2, b1));
                    const float2 nb1 = __ffma2_rn(c2, b1, __fmul2_rn(m2, b0));
                    const float2 nc0 = __ffma2_rn(c2, c0, __fmul2_rn(s2, c1));
                    const float2 nc1 = __ffma2_rn(c2, c1, __fmul2_rn(m2, c0));
                    store(jj, r, pack_bf16x2(nb0.x, nb1.x), pack_bf16x2(nc0.x, nc1.x));
                    store(jj + 1, r, pack_bf16x2(nb0.y, nb1.y), pack_bf16x2(nc0.y, nc1.y));
                }
            }
            if constexpr (TPT % 2 == 1) {
                const int jj = TPT - 1;
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    float b0 = bf16lo(bv[jj][r]), b1 = bf16hi(bv[jj][r]);
                    float c0 = bf16lo(cv[jj][r]), c1 = bf16hi(cv[jj][r]);
                    if constexpr (bc) {
                        b0 = fmaf(b0, sb[jj][r], bb0);
                        b1 = fmaf(b1, sb[jj][r], bb1);
                        c0 = fmaf(c0, sc[jj][r], cb0);
                        c1 = fmaf(c1, sc[jj][r], cb1);
                    }
                    store(jj, r, pack_bf16x2(fmaf(cn[jj], b0, sn[jj] * b1), fmaf(cn[jj], b1, -sn[jj] * b0)),
                          pack_bf16x2(fmaf(cn[jj], c0, sn[jj] * c1), fmaf(cn[jj], c1, -sn[jj] * c0)));
                }
            }
            }
            psi_acc += tot;
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar[RAW_EMPTY0 + rs]);
        }
        const int cs = c % kCoefSlots;
        Coef<NST, Q, R> cf{reinterpret_cast<float*>(sm + C::OFF_COEF) + cs * C::COEF_FLOATS};
        psi_acc -= 6.283185307179586f * rintf(psi_acc * 0.15915494309189535f);
        if (ts == 0) cf.psi_end()[pair] = psi_acc;

        // ---- w-scaled X:  Xw[u, r] = 2^(cum2_end - cum2_u) w_u x[u, r]  (needs the
        //      coefficient warp's decay prefix sums of this chunk)
        if (!warp_wait(&bar[CUM_READY0 + cs], (c / kCoefSlots) & 1, ab)) return;
        const int xs = c % C::XST;
        if (!warp_wait(&bar[X_FULL0 + xs], (c / C::XST) & 1, ab)) return;
        {
            const uint8_t* xt = sm + C::OFF_X + xs * C::X_BYTES;
            uint8_t* xw = C::xw(sm, slot);
            const float cend = *cf.cum2_end();
#pragma unroll 2
            for (int idx = tid; idx < C::L * 8; idx += 32 * kRotWarps) {
                const int row = idx >> 3, ch = idx & 7;
                const int u = row / R;
                const float sc = ex2_approx(cend - cf.cum2()[u]) * cf.w()[u];
                const uint32_t off = (uint32_t)row * 128u + ((uint32_t)((ch ^ row) & 7) << 4);
                uint4 v = *reinterpret_cast<const uint4*>(xt + off);
                // on the packed bf16 pairs: the weight is rounded to bf16 once
                const __nv_bfloat162 s2 = __float2bfloat162_rn(sc);
                auto mul = [&](uint32_t u) {
                    const __nv_bfloat162 t = __hmul2(*reinterpret_cast<const __nv_bfloat162*>(&u), s2);
                    return *reinterpret_cast<const uint32_t*>(&t);
                };
                *reinterpret_cast<uint4*>(xw + off) = make_uint4(mul(v.x), mul(v.y), mul(v.z), mul(v.w));
            }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
            mbar_arrive(&bar[COEF_FULL0 + cs]);
            mbar_arrive(&bar[OPS_FULL0 + slot]);
            mbar_arrive(&bar[DT_EMPTY0 + st]);
        }
    }
}

// Coefficient warp: per-token log2-decay prefix sum (warp scan), gamma, w and the mask
// exponent offsets ew_u = log2(w_u) - cum2_u of each chunk, into a ring of slots.
template <int NST, int Q, int R, bool GT>
__device__ void coefficients(const TcParams& p, const Unit& u, uint8_t* sm, uint64_t* bar,
                             const Abort& ab) {
    using C = Cfg<NST, Q, R, GT>;
    const int lane = threadIdx.x & 31;
    const int hq = u.h & 3;
    for (int c = 0; c < u.nch; ++c) {
        // tokens at or past the segment end lend no beta term to the last token: its
        // w is gamma alone, as at the end of the call
        const long long tnext = u.t0 + (long long)c * Q + 1;
        const int st = c & 1, cs = c % kCoefSlots;
        if (!warp_wait(&bar[DT_FULL0 + st], (c >> 1) & 1, ab)) return;
        const float* dtt = reinterpret_cast<const float*>(sm + C::OFF_DT + st * 3 * C::DT_BYTES);
        const float* At = dtt + C::DT_BYTES / 4;
        const float* lt = dtt + 2 * C::DT_BYTES / 4;
        Coef<NST, Q, R> cf{reinterpret_cast<float*>(sm + C::OFF_COEF) + cs * C::COEF_FLOATS};
        if (!warp_wait(&bar[COEF_EMPTY0 + cs], ((c / kCoefSlots) & 1) ^ 1, ab)) return;
        float carry = 0.f;
        for (int t0 = 0; t0 < Q; t0 += 32) {
            const int t = t0 + lane;
            float l2 = 0.f, gm = 0.f, wv = 0.f;
            if (t < Q) {
                const float d = dtt[t * 4 + hq], lm = lt[t * 4 + hq];
                l2 = d * At[t * 4 + hq] * kLog2e;
                gm = lm * d;
                const float dn = tnext + t < u.tend ? dtt[(t + 1) * 4 + hq] : 0.f;
                const float ln = lt[(t + 1) * 4 + hq];
                wv = gm + (1.f - ln) * dn;
            }
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float v = __shfl_up_sync(0xffffffffu, l2, o);
                if (lane >= o) l2 += v;
            }
            l2 += carry;
            if (t < Q) {
                cf.cum2()[t] = l2;
                cf.gam()[t] = gm;
                cf.w()[t] = wv;
                cf.ew()[t] = __log2f(wv) - l2;   // -inf when w = 0: the mask entry is 0
            }
            carry = __shfl_sync(0xffffffffu, l2, 31);
        }
        if (lane == 0) *cf.cum2_end() = carry;
        __syncwarp();
        if (lane == 0) {
            mbar_arrive(&bar[CUM_READY0 + cs]);
            mbar_arrive(&bar[COEF_FULL0 + cs]);
            mbar_arrive(&bar[DT_EMPTY0 + st]);
        }
    }
}

// ---------------------------------------------------------------------------------
// TMEM lane layouts of the epilogue and state warpgroups (warp w reaches lane quadrant
// w % 4).  Rows of an M = 128 accumulator: row 32q + lane, all columns.  Rows of an
// M = 64 accumulator: row 16q + lane % 16, column half lane / 16.  TMEM is read and
// written 16 of a thread's columns at a time.
template <int NST, int Q, int R>
struct Lanes {
    uint32_t tq;    // TMEM address of this warp's lane quadrant
    int lane, q;
    __device__ Lanes(uint32_t tmem) {
        lane = threadIdx.x & 31;
        q = (threadIdx.x >> 5) & 3;
        tq = tmem + ((uint32_t)(32 * q) << 16);
    }
    __device__ int row(bool half) const { return half ? 16 * q + (lane & 15) : 32 * q + lane; }
    __device__ int col0(bool half) const { return half ? 32 * (lane >> 4) : 0; }
    __device__ void ld16(bool half, uint32_t col, int cb, uint32_t (&v)[16]) const {
        if (half)
            tmem_ld_16x32bx2_x16<32>(tq + col + cb, v);
        else
            tmem_ld_32x32b_x16(tq + col + cb, v);
    }
    __device__ void st16(bool half, uint32_t col, int cb, const uint32_t (&v)[16]) const {
        if (half)
            tmem_st_16x32bx2_x16<32>(tq + col + cb, v);
        else
            tmem_st_32x32b_x16(tq + col + cb, v);
    }
};

// Epilogue warpgroup (warps 2-5): masks S into the bf16 operand S o L and writes y.
template <int NST, int Q, int R, bool GT>
__device__ void epilogue(const TcParams& p, const Unit& u, uint8_t* sm, uint64_t* bar,
                         uint32_t tmem, const Abort& ab) {
    using C = Cfg<NST, Q, R, GT>;
    const ScanArgs& a = p.a;
    const Lanes<NST, Q, R> ln(tmem);
    const int lane = ln.lane;
    const int etid = threadIdx.x - 64;                     // 0..127
    const float Dh = a.D ? a.D[u.h] : 0.f;
    constexpr bool kHalfL = (C::L == 64);
    const int lrow = ln.row(kHalfL), lcol0 = ln.col0(kHalfL);
    constexpr int kLCols = kHalfL ? 32 : C::L;
    constexpr int kYCols = kHalfL ? 32 : kP;
    uint8_t* sl = sm + C::OFF_SL;

    for (int c = 0; c < u.nch; ++c) {
        const uint32_t ph = c & 1, ph2 = (c >> 1) & 1;
        const int cs = c % kCoefSlots;
        Coef<NST, Q, R> cf{reinterpret_cast<float*>(sm + C::OFF_COEF) + cs * C::COEF_FLOATS};
        if (!warp_wait(&bar[COEF_FULL0 + cs], (c / kCoefSlots) & 1, ab)) return;
        const float* cum2 = cf.cum2();

        // ---- S o L -> bf16, K-major [row][col].  L[t,u] = 2^(cum2_t + ew_u) for u < t
        //      (ew_u = log2 w_u - cum2_u), gamma_t on the diagonal token; the skip D x is
        //      folded in as D on the (row == col) diagonal.
        if (!warp_wait(&bar[S_FULL], ph, ab)) return;
        tc_fence_after();
        {
            const int t = lrow / R;
            const float ct = cum2[t];
            const float gt = cf.gam()[t];
            const float* ew = cf.ew();
            const int tR = t * R;                  // first column of the row's own token
#pragma unroll 1
            for (int cb = 0; cb < kLCols; cb += 16) {
                uint32_t sv[16];
                ln.ld16(kHalfL, C::TM_S, cb, sv);
                tmem_wait_ld();
                const int colb = lcol0 + cb;
#pragma unroll
                for (int j = 0; j < 16; j += 8) {
                    float m[8];
                    // the R columns of one token share their mask value (colb + j is a
                    // multiple of 8, so of R): one exp2 per token, not per column
#pragma unroll
                    for (int e0 = 0; e0 < 8; e0 += R) {
                        const int u = (colb + j + e0) / R;
                        const float lv = ex2_approx(ct + ew[u]);
#pragma unroll
                        for (int rr = 0; rr < R; ++rr) {
                            const int e = e0 + rr, col = colb + j + e;
                            const float sv_f = __uint_as_float(sv[j + e]);
                            // earlier tokens: decay times the trapezoid weight; the own
                            // token's R columns: gamma (plus D on the diagonal); later: 0
                            const float d = fmaf(sv_f, gt, col == lrow ? Dh : 0.f);
                            m[e] = col < tR ? sv_f * lv : (col < tR + R ? d : 0.f);
                        }
                    }
                    uint4 o;
                    o.x = pack_bf16x2(m[0], m[1]);
                    o.y = pack_bf16x2(m[2], m[3]);
                    o.z = pack_bf16x2(m[4], m[5]);
                    o.w = pack_bf16x2(m[6], m[7]);
                    const int col = colb + j;
                    *reinterpret_cast<uint4*>(sl + (col >> 6) * C::L * 128 +
                                              sw128_off(lrow, col & 63)) = o;
                }
            }
        }
        tc_fence_before();
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
            mbar_arrive(&bar[S_EMPTY]);
            mbar_arrive(&bar[SL_FULL]);
        }

        // ---- y = Y_intra + e^{cum_t} Y_inter   (D x is in Y_intra; y is written over the
        //      x tile, which the x warp then stores with TMA)
        const int yb = c & 1;
        if (!warp_wait(&bar[Y_FULL0 + yb], ph2, ab)) return;
        const int xs = c % C::XST;
        if (!warp_wait(&bar[X_FULL0 + xs], (c / C::XST) & 1, ab)) return;
        tc_fence_after();
        uint8_t* xt = sm + C::OFF_X + xs * C::X_BYTES;
        const uint8_t* zt = sm + C::OFF_Z + xs * C::X_BYTES;   // z tile (gate only)
        {
            const float sc = exp2f(cum2[lrow / R]);
#pragma unroll 1
            for (int cb = 0; cb < kYCols; cb += 16) {
                uint32_t ya[16], yi[16];
                ln.ld16(kHalfL, C::tm_ya(yb), cb, ya);
                ln.ld16(kHalfL, C::tm_yi(yb), cb, yi);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 16; j += 8) {
                    const uint32_t off = sw128_off(lrow, lcol0 + cb + j);
                    float v[8];
#pragma unroll
                    for (int e = 0; e < 8; e += 2) {   // packed fp32x2: two columns per FMA
                        const float2 r2 = __ffma2_rn(
                            make_float2(sc, sc),
                            make_float2(__uint_as_float(yi[j + e]), __uint_as_float(yi[j + e + 1])),
                            make_float2(__uint_as_float(ya[j + e]), __uint_as_float(ya[j + e + 1])));
                        v[e] = r2.x;
                        v[e + 1] = r2.y;
                    }
                    if constexpr (GT) {
                        // the z tile has the x tile's layout: same swizzled offset
                        const uint4 zq = *reinterpret_cast<const uint4*>(zt + off);
                        const uint32_t zw[4] = {zq.x, zq.y, zq.z, zq.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            v[2 * e] *= silu_fast(bf16lo(zw[e]));
                            v[2 * e + 1] *= silu_fast(bf16hi(zw[e]));
                        }
                    }
                    uint32_t o[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) o[e] = pack_bf16x2(v[2 * e], v[2 * e + 1]);
                    *reinterpret_cast<uint4*>(xt + off) = make_uint4(o[0], o[1], o[2], o[3]);
                }
            }
        }
        tc_fence_before();
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
            mbar_arrive(&bar[Y_EMPTY0 + yb]);
            mbar_arrive(&bar[Y_STAGED0 + xs]);
        }
    }
}

// State warpgroup (warps 16-19): the fp32 carried state g in TMEM columns TM_G..,
// g_0 = h0 + (1 - lam_0) dt_0 B_prev x_prev^T, per chunk g <- e^{cum_end} g + dS and its
// bf16 copy for the Y_inter MMA; at the end h_T = R(psi_T) g and the carried x.
// Segmented calls: the segment pass (MAP) starts segment s from h0 (s = 0) or from no
// state (s > 0) plus the beta term of its first token, whose previous token is then the
// call's token t0 - 1; it records that g_0 and, instead of h_T, the segment's final
// state, total decay and final angles.  The output pass starts from the recorded g_0
// (completed by the chain step), and only the last segment writes h_T and the carried x.
template <int NST, int Q, int R, bool GT, bool BC, bool XE, bool MAP>
__device__ void state(const TcParams& p, const Unit& u, uint8_t* sm, uint64_t* bar,
                      uint32_t tmem, const Abort& ab) {
    using C = Cfg<NST, Q, R, GT>;
    const ScanArgs& a = p.a;
    const Lanes<NST, Q, R> ln(tmem);
    const int lane = ln.lane;
    const int stid = threadIdx.x - 512;                    // 0..127
    const int b = u.b, h = u.h, g = u.g;
    const long long T = a.T;
    const size_t bh = u.bh;
    constexpr bool kHalfN = (NST == 64);
    const int nrow = ln.row(kHalfN), ncol0 = ln.col0(kHalfN);
    constexpr int kNCols = kHalfN ? 32 : kP;
    uint8_t* gs = sm + C::OFF_G;
    float* rec = p.S > 1 ? p.seg + ((size_t)u.s * a.batch * a.H + bh) * seg_rec_floats(NST, kP)
                         : nullptr;

    auto publish16 = [&](int cb, const uint32_t (&v)[16]) {
#pragma unroll
        for (int j = 0; j < 16; j += 8) {
            uint4 o;
            o.x = pack_bf16x2(__uint_as_float(v[j]), __uint_as_float(v[j + 1]));
            o.y = pack_bf16x2(__uint_as_float(v[j + 2]), __uint_as_float(v[j + 3]));
            o.z = pack_bf16x2(__uint_as_float(v[j + 4]), __uint_as_float(v[j + 5]));
            o.w = pack_bf16x2(__uint_as_float(v[j + 6]), __uint_as_float(v[j + 7]));
            *reinterpret_cast<uint4*>(gs + sw128_off(nrow, ncol0 + cb + j)) = o;
        }
    };

    // ---- g_0 = h0 + (1 - lam_t0) dt_t0 B_prev x_prev^T
    {
        const bool prepared = !MAP && p.S > 1;   // recorded by the segment pass and the chain
        const bool carried = u.s == 0;           // the previous token is the carried one
        const size_t tok0 = (size_t)b * T + u.t0;  // the segment's first token
        const float d0 = a.dt[tok0 * a.H + h], l0 = a.lam[tok0 * a.H + h];
        const float beta0 = (1.f - l0) * d0;
        const __nv_bfloat16* bp =
            carried ? static_cast<const __nv_bfloat16*>(a.B_prev) + ((size_t)b * a.G + g) * R * NST
                    : static_cast<const __nv_bfloat16*>(a.B) + ((tok0 - 1) * a.G + g) * R * NST;
        // BCNorm scale of the previous token's B (rank r): the carried token's, or the
        // call's token t0 - 1
        const size_t Tp = (size_t)bc_tpad(T);
        auto bscale = [&](int r) -> float {
            if (!a.bc_scale) return 1.f;
            return carried ? a.bc_scale[2 * (size_t)a.batch * a.G * R * Tp +
                                        ((size_t)b * a.G + g) * R + r]
                           : a.bc_scale[(((size_t)b * a.G + g) * R + r) * Tp + (u.t0 - 1)];
        };
        // the previous token's X: the carried (already expanded) x, or the call's x at
        // t0 - 1, expanded and rounded as the x stages hold it
        const float* wx = (!carried && XE && a.x_expand) ? a.x_expand + (size_t)h * R * kP : nullptr;
        const __nv_bfloat16* xp =
            carried ? static_cast<const __nv_bfloat16*>(a.x_prev) + bh * R * kP
                    : static_cast<const __nv_bfloat16*>(a.x) + ((tok0 - 1) * a.H + h) * (wx ? 1 : R) * kP;
        auto xval = [&](int r, int col) -> float {
            if (wx)
                return __bfloat162float(
                    __float2bfloat16_rn(__bfloat162float(xp[col]) * wx[r * kP + col]));
            return __bfloat162float(xp[r * kP + col]);
        };
        const float* Bb = a.B_bias ? a.B_bias + (size_t)h * NST : nullptr;
        const float* h0 = a.h + (bh * NST + nrow) * kP + ncol0;
        float* g0r = rec ? rec + seg_off_g0(NST, kP) + (size_t)nrow * kP + ncol0 : nullptr;
#pragma unroll 1
        for (int cb = 0; cb < kNCols; cb += 16) {
            float gv[16];
            if (prepared) {
#pragma unroll
                for (int j = 0; j < 16; j += 4) {
                    const float4 v = *reinterpret_cast<const float4*>(g0r + cb + j);
                    gv[j] = v.x; gv[j + 1] = v.y; gv[j + 2] = v.z; gv[j + 3] = v.w;
                }
            } else {
                // the segment pass starts a later segment from no state
#pragma unroll
                for (int j = 0; j < 16; j += 4) {
                    const float4 v = carried ? *reinterpret_cast<const float4*>(h0 + cb + j)
                                             : make_float4(0.f, 0.f, 0.f, 0.f);
                    gv[j] = v.x; gv[j + 1] = v.y; gv[j + 2] = v.z; gv[j + 3] = v.w;
                }
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    const float bv0 = __bfloat162float(bp[r * NST + nrow]);
                    const float bb = beta0 * (BC ? bc_apply(bv0, bscale(r), Bb, nrow) : bv0);
#pragma unroll
                    for (int j = 0; j < 16; ++j) gv[j] = fmaf(bb, xval(r, ncol0 + cb + j), gv[j]);
                }
                if (MAP) {
#pragma unroll
                    for (int j = 0; j < 16; j += 4)
                        *reinterpret_cast<float4*>(g0r + cb + j) =
                            make_float4(gv[j], gv[j + 1], gv[j + 2], gv[j + 3]);
                }
            }
            uint32_t v[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) v[j] = __float_as_uint(gv[j]);
            ln.st16(kHalfN, C::TM_G, cb, v);
            if constexpr (!MAP) publish16(cb, v);
        }
        tmem_wait_st();
        if constexpr (!MAP) {
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar[G_FULL]);
        }
    }

    float cum_seg = 0.f;   // the segment's summed log2-decay (segment pass)
    for (int c = 0; c < u.nch; ++c) {
        const uint32_t ph = c & 1;
        const int cs = c % kCoefSlots;
        Coef<NST, Q, R> cf{reinterpret_cast<float*>(sm + C::OFF_COEF) + cs * C::COEF_FLOATS};
        if (!warp_wait(&bar[COEF_FULL0 + cs], (c / kCoefSlots) & 1, ab)) return;
        if (!warp_wait(&bar[DS_FULL], ph, ab)) return;
        const bool more = c + 1 < u.nch;
        // the Y_inter MMA of this chunk must be done reading g_c before g_{c+1} replaces it
        if (!MAP && more && !warp_wait(&bar[G_EMPTY], ph, ab)) return;
        tc_fence_after();
        const float c2e = *cf.cum2_end();
        const float dec = exp2f(c2e);
        cum_seg += c2e;
        if (c + 1 == u.nch) {
            // last chunk: the final state goes back to the original frame,
            // h_T = R(psi_T) (e^{cum_end} g + dS): the call's h_T (its last segment), or the
            // segment's final state of the segment pass
            float* out = MAP ? rec + (size_t)nrow * kP + ncol0
                             : (u.last ? a.h + (bh * NST + nrow) * kP + ncol0 : nullptr);
            float sn, cn;
            sincosf(cf.psi_end()[nrow >> 1], &sn, &cn);
            const bool odd = nrow & 1;
            if (out) {
#pragma unroll 1
                for (int cb = 0; cb < kNCols; cb += 16) {
                    uint32_t d[16], gq[16];
                    ln.ld16(kHalfN, C::TM_DS, cb, d);
                    ln.ld16(kHalfN, C::TM_G, cb, gq);
                    tmem_wait_ld();
                    float gv[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const float gj = fmaf(dec, __uint_as_float(gq[j]), __uint_as_float(d[j]));
                        const float o = __shfl_xor_sync(0xffffffffu, gj, 1);
                        gv[j] = odd ? fmaf(sn, o, cn * gj) : fmaf(cn, gj, -sn * o);
                    }
#pragma unroll
                    for (int j = 0; j < 16; j += 4)
                        *reinterpret_cast<float4*>(out + cb + j) =
                            make_float4(gv[j], gv[j + 1], gv[j + 2], gv[j + 3]);
                }
            }
            if (MAP) {
                if (!odd && ncol0 == 0) rec[seg_off_psi(NST, kP) + (nrow >> 1)] = cf.psi_end()[nrow >> 1];
                if (stid == 0) rec[seg_off_dec(NST, kP)] = exp2f(cum_seg);
            }
        } else {
#pragma unroll 1
            for (int cb = 0; cb < kNCols; cb += 16) {
                uint32_t d[16], gq[16];
                ln.ld16(kHalfN, C::TM_DS, cb, d);
                ln.ld16(kHalfN, C::TM_G, cb, gq);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 16; j += 2) {   // packed fp32x2: two columns per FMA
                    const float2 r2 = __ffma2_rn(
                        make_float2(dec, dec),
                        make_float2(__uint_as_float(gq[j]), __uint_as_float(gq[j + 1])),
                        make_float2(__uint_as_float(d[j]), __uint_as_float(d[j + 1])));
                    gq[j] = __float_as_uint(r2.x);
                    gq[j + 1] = __float_as_uint(r2.y);
                }
                ln.st16(kHalfN, C::TM_G, cb, gq);
                if constexpr (!MAP) publish16(cb, gq);
            }
            tmem_wait_st();
        }
        tc_fence_before();
        if constexpr (!MAP) fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
            mbar_arrive(&bar[DS_EMPTY]);
            if (!MAP && more) mbar_arrive(&bar[G_FULL]);
            mbar_arrive(&bar[COEF_EMPTY0 + cs]);   // this warp has read the slot's cum2_end
        }
    }
    if (!MAP && u.last && stid == 0) {
        // only this warpgroup read x_prev (for g_0, and in a segmented call the segment
        // pass read it before this launch), so the carried x can be replaced now; with the
        // lightweight expansion it takes the expanded X_{T-1}, as the stage held it
        const size_t row = ((size_t)b * T + (T - 1)) * a.H + h;
        if (XE && a.x_expand) {
            const __nv_bfloat16* xl = static_cast<const __nv_bfloat16*>(a.x) + row * kP;
            const float* wxl = a.x_expand + (size_t)h * R * kP;
            __nv_bfloat16* xpo = static_cast<__nv_bfloat16*>(a.x_prev) + bh * R * kP;
            for (int e = 0; e < R * kP; ++e)
                xpo[e] = __float2bfloat16_rn(__bfloat162float(xl[e % kP]) * wxl[e]);
        } else {
            const uint4* xl = reinterpret_cast<const uint4*>(
                static_cast<const __nv_bfloat16*>(a.x) + row * R * kP);
            uint4* xpo = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.x_prev) + bh * R * kP);
            for (int e = 0; e < R * kP / 8; ++e) xpo[e] = xl[e];
        }
    }
}

// Wait for a barrier phase with a fixed time limit, regardless of the abort flag
// (used on the way out, to let in-flight copies and MMAs land before exiting).
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity, uint64_t ns) {
    const uint64_t t0 = globaltimer();
    while (!mbar_try_wait(bar, parity) && globaltimer() - t0 < ns) {
    }
}

template <int NST, int Q, int R, bool GT, bool BC, bool MAP>
__device__ void producer(const TcParams& p, const Unit& u, uint8_t* sm, uint64_t* bar,
                         const Abort& ab) {
    using C = Cfg<NST, Q, R, GT>;
    const ScanArgs& a = p.a;
    const int b = u.b, h = u.h, g = u.g;
    // loads issued per ring stage, so that an aborted CTA can wait for them to land
    int n_dt[2] = {0, 0}, n_raw[2] = {0, 0};
    int raw_it = 0;
    bool ok = true;
    for (int c = 0; c < u.nch && ok; ++c) {
        const int t0 = (int)(u.t0 + (long long)c * Q), st = c & 1;
        const uint32_t ph = ((c >> 1) & 1) ^ 1;
        // per-chunk dt / A / lam (Q+1 tokens: the next chunk's first token is the lookahead)
        if (!(ok = mbar_wait(&bar[DT_EMPTY0 + st], ph, ab))) break;
        mbar_arrive_expect_tx(&bar[DT_FULL0 + st], 3 * C::DT_BOX);
        float* dtt = reinterpret_cast<float*>(sm + C::OFF_DT + st * 3 * C::DT_BYTES);
        tma_load_3d(dtt, &p.tm_dt, &bar[DT_FULL0 + st], h & ~3, t0, b);
        tma_load_3d(dtt + C::DT_BYTES / 4, &p.tm_A, &bar[DT_FULL0 + st], h & ~3, t0, b);
        tma_load_3d(dtt + 2 * C::DT_BYTES / 4, &p.tm_lam, &bar[DT_FULL0 + st], h & ~3, t0, b);
        ++n_dt[st];
        // raw B, C, theta in sub-chunks of RT tokens; the x tile after the first one
        for (int s = 0; s < C::NSUB; ++s, ++raw_it) {
            const int rs = raw_it & 1;
            if (!(ok = mbar_wait(&bar[RAW_EMPTY0 + rs], ((raw_it >> 1) & 1) ^ 1, ab))) break;
            const bool sc = BC && a.bc_scale != nullptr;
            // the segment pass reads no C
            mbar_arrive_expect_tx(&bar[RAW_FULL0 + rs],
                                  C::SC_OFF - (MAP ? C::BRAW_BYTES : 0) + (sc ? C::SC_BOX : 0));
            uint8_t* raw = sm + C::OFF_RAW + rs * C::RAW_BYTES;
            const int tr = t0 + s * C::RT;
            tma_load_5d(raw, &p.tm_B, &bar[RAW_FULL0 + rs], 0, 0, g, tr, b);
            if (!MAP)
                tma_load_5d(raw + C::BRAW_BYTES, &p.tm_C, &bar[RAW_FULL0 + rs], 0, 0, g, tr, b);
            tma_load_4d(raw + 2 * C::BRAW_BYTES, &p.tm_th, &bar[RAW_FULL0 + rs], 0, g, tr, b);
            if (sc)   // BCNorm scales of B and C for these tokens: x = token (RT-aligned)
                tma_load_5d(raw + C::SC_OFF, &p.tm_sc, &bar[RAW_FULL0 + rs], tr, 0, g, b, 0);
            ++n_raw[rs];
        }
    }
    if (!ok) {
        // aborted: let every load already issued land before the CTA exits
        for (int s = 0; s < 2; ++s) {
            if (n_dt[s]) drain_wait(&bar[DT_FULL0 + s], (n_dt[s] - 1) & 1, 10000000ull);
            if (n_raw[s]) drain_wait(&bar[RAW_FULL0 + s], (n_raw[s] - 1) & 1, 10000000ull);
        }
    }
}

// x tiles and y stores, on their own warp so that neither a stage waiting for its y
// store nor the store itself holds up the B / C / theta loads.  x(c) is loaded into
// stage c % XST; once the epilogue has written y(c) over it (Y_STAGED), the tile is
// stored, and when the store has read it the stage takes x(c + XST).  In the segment pass
// nothing is stored: Y_STAGED then says the rotation warps are done with x(c).
//
// MIMO lightweight expansion ("Multi-Input, Multi-Output (MIMO) Formulation", MIMO
// Parameterization Choices): x (and z) then hold one value per head channel, and the
// stage's (token, rank) row is X[u, r][p] = x_u[p] w[r][p], rounded to bf16.  The chunk's
// Q raw rows are copied, unswizzled, into the stage's last Q rows and expanded in place by
// the whole warp, token batch after token batch: every lane reads its batch before any
// lane writes it, and the rows a batch writes, [t0 R, (t0 + k) R), lie below the raw row
// (R - 1) Q + t0 + k of the first later token because (t0 + k)(R - 1) <= Q (R - 1).  The
// stage is published on X_FULL once expanded.
template <int NST, int Q, int R, bool GT, bool XE, bool MAP>
__device__ void x_producer(const TcParams& p, const Unit& u, uint8_t* sm, uint64_t* bar,
                           const Abort& ab) {
    using C = Cfg<NST, Q, R, GT>;
    const ScanArgs& a = p.a;
    const int lane = threadIdx.x & 31;
    const int b = u.b, h = u.h;
    // token coordinate of chunk c of the segment
    auto tok = [&](int c) { return (int)(u.t0 + (long long)c * Q); };
    if constexpr (!XE) {   // lane 0 alone: every tile comes by TMA
        if (lane != 0) return;
        int n_x[C::XST] = {};
        auto load = [&](int c) {
            const int xs = c % C::XST;
            mbar_arrive_expect_tx(&bar[X_FULL0 + xs], C::XZ_BYTES);
            tma_load_5d(sm + C::OFF_X + xs * C::X_BYTES, &p.tm_x, &bar[X_FULL0 + xs], 0, 0, h,
                        tok(c), b);
            if constexpr (GT)
                tma_load_5d(sm + C::OFF_Z + xs * C::X_BYTES, &p.tm_z, &bar[X_FULL0 + xs], 0, 0, h,
                            tok(c), b);
            ++n_x[xs];
        };
        for (int c = 0; c < C::XST && c < u.nch; ++c) load(c);
        bool ok = true;
        for (int c = 0; c < u.nch; ++c) {
            if (!(ok = mbar_wait(&bar[Y_STAGED0 + c % C::XST], (c / C::XST) & 1, ab))) break;
            const int xs = c % C::XST;
            if constexpr (!MAP) {
                tma_store_5d(&p.tm_y, sm + C::OFF_X + xs * C::X_BYTES, 0, 0, h, tok(c), b);
                bulk_commit();
            }
            mbar_arrive(&bar[COEF_EMPTY0 + c % kCoefSlots]);
            if constexpr (!MAP) bulk_wait_read<0>();
            if (c + C::XST < u.nch) load(c + C::XST);
        }
        if (!ok)
            for (int s = 0; s < C::XST; ++s)
                if (n_x[s]) drain_wait(&bar[X_FULL0 + s], (n_x[s] - 1) & 1, 10000000ull);
        bulk_wait<0>();
        return;
    } else {
    const bool xe = a.x_expand != nullptr, ze = GT && a.z_expand != nullptr;
    // expansion: lane = (rank r, 16-byte column chunk ch) for TPL tokens side by side
    constexpr int CMB = 8 * R, TPL = 32 / CMB;
    static_assert(32 % CMB == 0 && Q % (2 * TPL) == 0, "expansion lane layout");
    const int r = (lane % CMB) >> 3, ch = lane & 7, toff = lane / CMB;
    // this lane's 8 weights w[r][8 ch .. 8 ch + 7] as 4 pairs (packed fp32x2 products)
    float2 wx[4], wz[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) wx[j] = wz[j] = make_float2(0.f, 0.f);
    if (xe) {
        const float2* w2 = reinterpret_cast<const float2*>(a.x_expand + ((size_t)h * R + r) * kP + 8 * ch);
#pragma unroll
        for (int j = 0; j < 4; ++j) wx[j] = w2[j];
    }
    if (ze) {
        const float2* w2 = reinterpret_cast<const float2*>(a.z_expand + ((size_t)h * R + r) * kP + 8 * ch);
#pragma unroll
        for (int j = 0; j < 4; ++j) wz[j] = w2[j];
    }
    auto mul2 = [](uint32_t v, float2 w) {   // two bf16 values times two weights, rounded
        const float2 p = __fmul2_rn(make_float2(bf16lo(v), bf16hi(v)), w);
        return pack_bf16x2(p.x, p.y);
    };
    // the stage's last Q rows (raw, unswizzled) -> its rows (u, r) (128B-swizzled), in place
    auto expand = [&](uint8_t* tile, const float2 (&w)[4]) {
        const uint8_t* raw = tile + (R - 1) * Q * 128;
#pragma unroll 1
        for (int t0 = 0; t0 < Q; t0 += 2 * TPL) {
            uint4 v[2];
#pragma unroll
            for (int k = 0; k < 2; ++k)
                v[k] = *reinterpret_cast<const uint4*>(raw + (t0 + k * TPL + toff) * 128 + ch * 16);
            __syncwarp();
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const int row = (t0 + k * TPL + toff) * R + r;
                const uint4 o = make_uint4(mul2(v[k].x, w[0]), mul2(v[k].y, w[1]),
                                           mul2(v[k].z, w[2]), mul2(v[k].w, w[3]));
                *reinterpret_cast<uint4*>(tile + row * 128 + (((ch ^ row) & 7) << 4)) = o;
            }
            __syncwarp();
        }
    };
    int n_xr = 0;           // copies issued on XR_FULL (each one phase)
    bool pending = false;   // a copy on XR_FULL has not been waited for
    // every copy of stage c lands on XR_FULL; the expanded stage is published on X_FULL
    auto load = [&](int c) -> bool {
        const int xs = c % C::XST;
        uint8_t* xt = sm + C::OFF_X + xs * C::X_BYTES;
        uint8_t* zt = sm + C::OFF_Z + xs * C::X_BYTES;
        if (lane == 0) {
            const int bytes = (xe ? Q * 128 : C::X_BYTES) + (GT ? (ze ? Q * 128 : C::X_BYTES) : 0);
            mbar_arrive_expect_tx(&bar[XR_FULL], bytes);
            if (xe)
                tma_load_4d(xt + (R - 1) * Q * 128, &p.tm_xr, &bar[XR_FULL], 0, h, tok(c), b);
            else
                tma_load_5d(xt, &p.tm_x, &bar[XR_FULL], 0, 0, h, tok(c), b);
            if constexpr (GT) {
                if (ze)
                    tma_load_4d(zt + (R - 1) * Q * 128, &p.tm_zr, &bar[XR_FULL], 0, h, tok(c), b);
                else
                    tma_load_5d(zt, &p.tm_z, &bar[XR_FULL], 0, 0, h, tok(c), b);
            }
        }
        pending = true;
        if (!warp_wait(&bar[XR_FULL], n_xr++ & 1, ab)) return false;
        pending = false;
        if (xe) expand(xt, wx);
        if (ze) expand(zt, wz);
        fence_proxy_async_smem();   // the expanded rows are read by the MMAs and the y store
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar[X_FULL0 + xs]);
        return true;
    };
    bool ok = true;
    for (int c = 0; c < C::XST && c < u.nch && ok; ++c) ok = load(c);
    for (int c = 0; c < u.nch && ok; ++c) {
        if (!(ok = warp_wait(&bar[Y_STAGED0 + c % C::XST], (c / C::XST) & 1, ab))) break;
        const int xs = c % C::XST;
        if (lane == 0) {
            if constexpr (!MAP) {
                tma_store_5d(&p.tm_y, sm + C::OFF_X + xs * C::X_BYTES, 0, 0, h, tok(c), b);
                bulk_commit();
            }
            mbar_arrive(&bar[COEF_EMPTY0 + c % kCoefSlots]);
            if constexpr (!MAP) bulk_wait_read<0>();
        }
        __syncwarp();
        if (c + C::XST < u.nch) ok = load(c + C::XST);
    }
    if (lane == 0) {
        if (pending) drain_wait(&bar[XR_FULL], (n_xr - 1) & 1, 10000000ull);
        bulk_wait<0>();
    }
    }
}

// MAP: the segment pass of a segmented call (no C~, S, Y or y; see Unit and state).
template <int NST, int Q, int R, bool GT, bool BC, bool XE, bool MAP>
__global__ void __launch_bounds__(kThreads, 1) scan_tc_kernel(const __grid_constant__ TcParams p) {
    using C = Cfg<NST, Q, R, GT>;
    const Unit u = unit_of<Q, MAP>(p);
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte aligned base for the SW128 tiles, as an offset from smem_raw so that the
    // compiler keeps every access in the shared address space
    uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + C::OFF_BAR);
    uint32_t* misc = reinterpret_cast<uint32_t*>(sm + C::OFF_MISC);
    const int w = threadIdx.x >> 5;

    if (threadIdx.x == 0) {
        for (int i = 0; i < NUM_BARS; ++i) mbar_init(&bar[i], bar_count(i));
        misc[1] = 0u;  // abort flag
        fence_mbar_init();
        tma_prefetch_desc(XE && p.a.x_expand ? &p.tm_xr : &p.tm_x);
        if (GT) tma_prefetch_desc(XE && p.a.z_expand ? &p.tm_zr : &p.tm_z);
        tma_prefetch_desc(&p.tm_B);
        if (!MAP) tma_prefetch_desc(&p.tm_C);
        tma_prefetch_desc(&p.tm_th);
        tma_prefetch_desc(&p.tm_dt);
    }
    if (w == 0) {
        tmem_alloc(&misc[0], kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc[0];
    Abort ab{reinterpret_cast<volatile uint32_t*>(&misc[1]), p.a.status, p.limit_ns};

    if (w == 0) {
        if ((threadIdx.x & 31) == 0) producer<NST, Q, R, GT, BC, MAP>(p, u, sm, bar, ab);
    } else if (w == 1) {
        if ((threadIdx.x & 31) == 0) {
            mma_issuer<NST, Q, R, GT, MAP>(p, u, sm, bar, tmem, ab);
            // no MMA may still be writing TMEM when it is released
            mma_commit(&bar[DRAIN]);
            drain_wait(&bar[DRAIN], 0, 100000000ull);
        }
    } else if (w < 6) {
        if constexpr (!MAP) epilogue<NST, Q, R, GT>(p, u, sm, bar, tmem, ab);
    } else if (w >= 16) {
        state<NST, Q, R, GT, BC, XE, MAP>(p, u, sm, bar, tmem, ab);
    } else if (w < 6 + kRotWarps) {
        rotation<NST, Q, R, GT, BC, MAP>(p, u, sm, bar, ab);
    } else if (w == 6 + kRotWarps) {
        coefficients<NST, Q, R, GT>(p, u, sm, bar, ab);
    } else if (XE || (threadIdx.x & 31) == 0) {
        x_producer<NST, Q, R, GT, XE, MAP>(p, u, sm, bar, ab);
    }
    tc_fence_before();
    __syncthreads();
    if (w == 0) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// Chain step between the segment pass and the output pass of a segmented call: the state
// entering segment s + 1 is dec_s R(psi_s) h_in(s) + M_s (M_0 already holds h0), and the
// output pass starts segment s from G0_s + h_in(s).  One thread per (batch * head, state
// pair, column), sequential over the segments.
__global__ void seg_chain_kernel(float* seg, int BH, int S, int N, int P) {
    const size_t rec = seg_rec_floats(N, P);
    const int per = (N / 2) * P;
    const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= (long long)BH * per) return;
    const int bh = (int)(idx / per), rem = (int)(idx % per), i = rem / P, col = rem % P;
    const size_t e0 = (size_t)(2 * i) * P + col, e1 = e0 + P;
    const float* r0 = seg + (size_t)bh * rec;
    float he = r0[e0], ho = r0[e1];   // the state entering segment 1
    for (int s = 1; s < S; ++s) {
        float* r = seg + ((size_t)s * BH + bh) * rec;
        float* g0 = r + seg_off_g0(N, P);
        g0[e0] += he;
        g0[e1] += ho;
        if (s + 1 < S) {
            const float dec = r[seg_off_dec(N, P)];
            float sn, cn;
            sincosf(r[seg_off_psi(N, P) + i], &sn, &cn);
            const float ne = fmaf(dec, fmaf(cn, he, -sn * ho), r[e0]);
            const float no = fmaf(dec, fmaf(sn, he, cn * ho), r[e1]);
            he = ne;
            ho = no;
        }
    }
}

// ---------------------------------------------------------------------------------
// host side: tensor maps and launch

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// cuTensorMapEncodeTiled from the driver, looked up once through the runtime (no -lcuda)
EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        cudaDriverEntryPointQueryResult q;
        void* ptr = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

bool make_map(CUtensorMap* m, CUtensorMapDataType dt, int rank, const void* ptr,
              const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box,
              CUtensorMapSwizzle swz) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    CUresult r = fn(m, dt, rank, const_cast<void*>(ptr), reinterpret_cast<const cuuint64_t*>(dims),
                    reinterpret_cast<const cuuint64_t*>(strides_bytes),
                    reinterpret_cast<const cuuint32_t*>(box), estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <int NST, int Q, int R, bool GT, bool BC, bool XE, bool MAP>
cudaError_t launch_k(const TcParams& p, unsigned grid, cudaStream_t s) {
    using C = Cfg<NST, Q, R, GT>;
    cudaError_t e = cudaFuncSetAttribute(scan_tc_kernel<NST, Q, R, GT, BC, XE, MAP>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    scan_tc_kernel<NST, Q, R, GT, BC, XE, MAP><<<grid, kThreads, C::SMEM, s>>>(p);
    return cudaGetLastError();
}

template <int NST, int Q, int R, bool GT, bool BC, bool XE>
cudaError_t launch_t(const ScanArgs& a, cudaStream_t s) {
    using C = Cfg<NST, Q, R, GT>;
    TcParams p;
    std::memset(&p, 0, sizeof(p));
    p.a = a;
    p.nch_total = (int)((a.T + Q - 1) / Q);
    p.limit_ns = (a.flags & M3_FLAG_TEST_STALL) ? 50000000ull : 2000000000ull;
    const uint64_t T = a.T, Bn = a.batch, H = a.H, G = a.G;
    bool ok = true;
    {   // x, y: (P, R, H, T, b), box (64, R, 1, Q, 1), 128B swizzle
        const uint64_t d[5] = {kP, R, H, T, Bn};
        const uint64_t st[4] = {kP * 2, (uint64_t)R * kP * 2, H * R * kP * 2, T * H * R * kP * 2};
        const uint32_t box[5] = {kP, R, 1, Q, 1};
        if (!a.x_expand)
            ok &= make_map(&p.tm_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, a.x, d, st, box,
                           CU_TENSOR_MAP_SWIZZLE_128B);
        ok &= make_map(&p.tm_y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, a.y, d, st, box,
                       CU_TENSOR_MAP_SWIZZLE_128B);
        if (GT && !a.z_expand)
            ok &= make_map(&p.tm_z, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, a.z, d, st, box,
                           CU_TENSOR_MAP_SWIZZLE_128B);
    }
    if (a.x_expand || (GT && a.z_expand)) {
        // x, z of the lightweight expansion: (P, H, T, b), box (64, 1, Q, 1), unswizzled rows
        const uint64_t d[4] = {kP, H, T, Bn};
        const uint64_t st[3] = {kP * 2, H * kP * 2, T * H * kP * 2};
        const uint32_t box[4] = {kP, 1, Q, 1};
        if (a.x_expand)
            ok &= make_map(&p.tm_xr, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, a.x, d, st, box,
                           CU_TENSOR_MAP_SWIZZLE_NONE);
        if (GT && a.z_expand)
            ok &= make_map(&p.tm_zr, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, a.z, d, st, box,
                           CU_TENSOR_MAP_SWIZZLE_NONE);
    }
    {   // B, C: (N, R, G, T, b), box (N, R, 1, RT, 1)
        const uint64_t d[5] = {NST, R, G, T, Bn};
        const uint64_t st[4] = {NST * 2, (uint64_t)R * NST * 2, G * R * NST * 2,
                                T * G * R * NST * 2};
        const uint32_t box[5] = {NST, R, 1, C::RT, 1};
        ok &= make_map(&p.tm_B, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, a.B, d, st, box,
                       CU_TENSOR_MAP_SWIZZLE_NONE);
        ok &= make_map(&p.tm_C, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, a.C, d, st, box,
                       CU_TENSOR_MAP_SWIZZLE_NONE);
    }
    {   // theta: (N/2, G, T, b), box (N/2, 1, RT, 1)
        const uint64_t d[4] = {NST / 2, G, T, Bn};
        const uint64_t st[3] = {NST / 2 * 4, G * NST / 2 * 4, T * G * NST / 2 * 4};
        const uint32_t box[4] = {NST / 2, 1, C::RT, 1};
        ok &= make_map(&p.tm_th, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, a.theta, d, st, box,
                       CU_TENSOR_MAP_SWIZZLE_NONE);
    }
    {   // dt, A, lam: (H, T, b), box (4, Q+1, 1)
        const uint64_t d[3] = {H, T, Bn};
        const uint64_t st[2] = {H * 4, T * H * 4};
        const uint32_t box[3] = {4, Q + 1, 1};
        ok &= make_map(&p.tm_dt, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, a.dt, d, st, box,
                       CU_TENSOR_MAP_SWIZZLE_NONE);
        ok &= make_map(&p.tm_A, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, a.A, d, st, box,
                       CU_TENSOR_MAP_SWIZZLE_NONE);
        ok &= make_map(&p.tm_lam, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, a.lam, d, st, box,
                       CU_TENSOR_MAP_SWIZZLE_NONE);
    }
    if (BC && a.bc_scale) {
        // BCNorm scales: (token, R, G, b, {B, C}) with rows of Tp tokens, box (RT, R, 1, 1, 2).
        // The token extent is T: the copy zero-fills past the end of the call.
        const uint64_t Tp = (uint64_t)bc_tpad(a.T);
        const uint64_t d[5] = {T, (uint64_t)R, G, Bn, 2};
        const uint64_t st[4] = {Tp * 4, (uint64_t)R * Tp * 4, G * R * Tp * 4, Bn * G * R * Tp * 4};
        const uint32_t box[5] = {(uint32_t)C::RT, (uint32_t)R, 1, 1, 2};
        ok &= make_map(&p.tm_sc, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 5, a.bc_scale, d, st, box,
                       CU_TENSOR_MAP_SWIZZLE_NONE);
    }
    if (!ok) return cudaErrorInvalidValue;
    // Sequence segments: when the workspace holds their records, the call runs as the
    // segment pass, the chain step and the output pass.
    const int BH = a.batch * a.H;
    int S = scan_tc_segments(BH, p.nch_total);
    const size_t seg_bytes = (size_t)BH * S * seg_rec_floats(NST, kP) * sizeof(float);
    if (S > 1 && (!a.ws || a.ws_bytes < seg_bytes)) S = 1;
    p.S = S;
    p.seg = S > 1 ? static_cast<float*>(a.ws) : nullptr;
    if (S > 1) {
        cudaError_t e = launch_k<NST, Q, R, false, BC, XE, true>(p, (unsigned)(BH * S), s);
        if (e != cudaSuccess) return e;
        const long long n = (long long)BH * (NST / 2) * kP;
        seg_chain_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(p.seg, BH, S, NST, kP);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    return launch_k<NST, Q, R, GT, BC, XE, false>(p, (unsigned)(BH * S), s);
}

}  // namespace


// The tile holds L = chunk * R (token, rank) rows with L in {64, 128}: the M = 64 / 128
// MMA shapes, and the S and Y accumulators that fit TMEM.  A requested chunk whose L
// falls outside is run with the nearest tile (L clamped into [64, 128]): the chunked form
// is exact for any blocking, so only rounding changes.  With N = 128 a 128-row tile
// leaves shared memory for a single operand slot, which serialises the rotation warps
// and the MMAs; chunk 128 then runs as 64-token tiles.  Returns 0 where no tile applies.
int scan_tc_chunk(int N, int P, int R, int chunk, int H) {
    if (P != kP || H % 4 != 0) return 0;
    if (R != 1 && R != 2 && R != 4) return 0;
    if (N != 64 && (N != 128 || R != 1)) return 0;
    int L = chunk * R;
    L = L < 64 ? 64 : (L > 128 ? 128 : L);
    if (N == 128) L = 64;
    return L / R;
}

// Segments per (batch, head) for a call of nch chunks over BH (batch * head) streams: one
// stream per SM of the current device, at least two chunks per segment, at most 16
// segments.  A segment pass chunk costs about 0.8 of an output pass chunk (measured on
// B200: 63 us for 32 chunks against 77 us), so two segments (1.8 / 2 of the time, before
// the chain step and the extra launches) do not pay: fewer than three means 1 (none).
int scan_tc_segments(int BH, long long nch) {
    // SM count per device, looked up once (the launch path calls this for every call)
    static int sms_of[64] = {};
    int sms = 148, dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess && dev >= 0 && dev < 64) {
        if (!sms_of[dev]) {
            int n = 0;
            if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess &&
                n > 0)
                sms_of[dev] = n;
        }
        if (sms_of[dev]) sms = sms_of[dev];
    }
    long long S = BH > 0 ? sms / BH : 1;
    if (S > nch / 2) S = nch / 2;
    if (S > 16) S = 16;
    return S < 3 ? 1 : (int)S;
}

// The segment records of a call that would be segmented (see scan_tc_segments); 0 otherwise.
size_t scan_tc_workspace_bytes(int batch, int H, int N, int P, int, long long T, int chunk) {
    const long long nch = (T + chunk - 1) / chunk;
    const int S = scan_tc_segments(batch * H, nch);
    return S > 1 ? (size_t)batch * H * S * seg_rec_floats(N, P) * sizeof(float) : 0;
}

template <bool GT, bool BC, bool XE>
cudaError_t launch_scan_tc_g(const ScanArgs& a, int R, cudaStream_t s) {
    const int N = a.N, Q = a.chunk;   // the tile chunk chosen by scan_tc_chunk
    if (R == 1) {
        if (N == 128 && Q == 64) return launch_t<128, 64, 1, GT, BC, XE>(a, s);
        if (N == 64 && Q == 64) return launch_t<64, 64, 1, GT, BC, XE>(a, s);
        if (N == 64 && Q == 128) return launch_t<64, 128, 1, GT, BC, XE>(a, s);
    } else if (R == 2 && N == 64) {
        if (Q == 32) return launch_t<64, 32, 2, GT, BC, XE>(a, s);
        if (Q == 64) return launch_t<64, 64, 2, GT, BC, XE>(a, s);
    } else if (R == 4 && N == 64) {
        if (Q == 16) return launch_t<64, 16, 4, GT, BC, XE>(a, s);
        if (Q == 32) return launch_t<64, 32, 4, GT, BC, XE>(a, s);
    }
    return cudaErrorNotSupported;
}

template <bool GT, bool BC>
cudaError_t launch_scan_tc_x(const ScanArgs& a, int R, cudaStream_t s) {
    const bool xe = a.x_expand || (GT && a.z_expand);
    return xe ? launch_scan_tc_g<GT, BC, true>(a, R, s) : launch_scan_tc_g<GT, BC, false>(a, R, s);
}

// a.z, a.bc and the expansion weights select the instantiation with the fused output gate,
// the BC map and the MIMO lightweight expansion
cudaError_t launch_scan_tc(const ScanArgs& a, int R, cudaStream_t s) {
    if (a.z) return a.bc ? launch_scan_tc_x<true, true>(a, R, s) : launch_scan_tc_x<true, false>(a, R, s);
    return a.bc ? launch_scan_tc_x<false, true>(a, R, s) : launch_scan_tc_x<false, false>(a, R, s);
}

}  // namespace m3
