// scan_bwd_tc.cu -- chunked backward pass of the Mamba-3 recurrence on the tensor cores
// (bf16 x / B / C / dy, P = 64; SISO with N in {64, 128}, MIMO ranks 2 and 4 with N = 64).
//
// Every tile has 64 rows; a row is one (token, rank), row = R u + r, so a chunk holds 64 / R
// tokens (the C_MIMO = C_SISO / R rule of "Expressing MIMO as Multiple SISO SSMs", "The
// Chunked Training Optimization").  Sums over a token's rows stand where the SISO formulas
// below have one row; every per-token factor (decay, weights, angle, causal mask) is looked up
// by row / R.
//
// Reverse-mode gradients of the chunked form ("Parallel representation under SSD", with the
// rotation of Propositions 3 and 4).  Per chunk [t0, t1) of Q = 64 / R tokens, with cum the prefix
// of the log-decays dt A, psi the prefix of the angles, B~ = R(-psi) B, C~ = R(-psi) C,
//     gamma_s = lam_s dt_s,   w_s = gamma_s + (1 - lam_{s+1}) dt_{s+1},
//     L[t, s] = e^{cum_t - cum_s} (gamma_s + [s < t] (1 - lam_{s+1}) dt_{s+1})    (s <= t),
// and g the state entering the chunk (in the rotated frame), the forward is
//     Y_t = e^{cum_t - m} C~_t g + sum_s L[t, s] (C~_t . B~_s) X_s + D X_t
//     g  <- e^{cum_end - m} g + sum_s e^{cum_end - cum_s} w_s B~_s X_s^T.
// The backward keeps the adjoint dg of g between chunks.  Four launches:
//   1. chunk products, per (batch, head, chunk): V = B~^T diag(e w) X and U = C~^T diag(f) dY
//      on the tensor cores (e_s = e^{cum_end - cum_s}, f_t = e^{cum_t - m}), in the chunk's own
//      frame (angles counted from the chunk start), with the chunk's total log-decay and angles;
//   2. chunk scan, per (batch, head): the state entering every chunk (forward) and the adjoint
//      of the state leaving it (reverse), turned into the call's frame and stored as bf16
//      operand tiles; the starting state's gradients and the dL/dh_T terms;
//   3. chunk gradients, per (batch, head, chunk), on the tensor cores: S = C~ B~^T and
//      dY X^T; the masked tiles L o S and dS = L o (dY X^T); then
//          dX  = (L o S)^T dY + diag(e w) B~ dg + D dY,
//          dC~ = dS B~ + diag(f) dY g^T,      dB~ = dS^T C~ + diag(e w) X dg^T,
//      rotated back by R(psi); the log-decay, band-weight and angle chains from row and
//      column sums of the same tiles;
//   4. carry, per (batch, head, pair): the angle gradient carried into every chunk from later
//      chunks; finish, per (batch, chunk, group): dtheta summed over the group's heads in a
//      fixed order, dt's angle term, and the next token's share of the trapezoid weight w of
//      the previous chunk's last token.
// Every reverse-mode term is the one the oracle's chunked route takes; the group-shared
// gradients B, C, B_prev and dD are added with atomics, so their last bits may vary from run
// to run.  Every wait is bounded; a timeout writes M3_ERR_TIMEOUT to the status word.
#include <cuda_bf16.h>

#include "m3_internal.h"
#include "sm100.cuh"

namespace m3 {

using namespace sm100;

namespace {

constexpr int kQ = 64;     // chunk tokens
constexpr int kPc = 64;    // head channels
constexpr float kTwoPi = 6.28318530717958647692f;
constexpr float kInvTwoPi = 0.15915494309189533577f;
constexpr float kLog2e = 1.44269504088896340736f;

struct TcBwd {
    BwdArgs a;
    int nch;                  // chunks of the call
    int qt;                   // tokens per chunk: 64 / R (a tile row is one (token, rank))
    uint16_t* V;              // [BH][nch][N][P] bf16 chunk-frame state products
    uint16_t* U;              // [BH][nch][N][P] bf16 chunk-frame adjoint products
    uint16_t* gin;            // [BH][nch] bf16 tile images [N][P] of the entering state
    uint16_t* dgo;            // [BH][nch] bf16 tile images [N][P] of the leaving adjoint
    float* ctot;              // [BH][nch] total log-decay of the chunk
    float* atot;              // [BH][nch][N/2] total angle of the chunk
    float* P0;                // [BH][nch + 1][N/2] angle before the chunk (mod 2 pi)
    float* q;                 // [BH][nch] e^{ctot} <dg_out, g_in>
    float* dtot;              // [BH][nch][N/2] sum of the chunk's angle gradients
    float* spill;             // [BH][nch] band-weight gradient owed to the next token
    float* extra;             // [BH][N/2] angle gradient of the last token from dL/dh_T
    float* pang;              // [BH][T][N/2] chunk-local suffix sums of the angle gradients
    float* carry;             // [BH][nch][N/2] angle gradient carried in from later chunks
    float* v0;                // [BH] <dg_0, B_prev x_prev^T>
    uint32_t* status;
    unsigned long long limit_ns;
};

__device__ __forceinline__ float wrap_angle(float x) {
    return fmaf(-kTwoPi, rintf(x * kInvTwoPi), x);
}
__device__ __forceinline__ float ex2f(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float bf_at(const void* base, size_t i) {
    return __uint_as_float((uint32_t)(static_cast<const uint16_t*>(base)[i]) << 16);
}
__device__ __forceinline__ uint16_t to_bf(float v) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(v));
}
__device__ __forceinline__ uint32_t scale2(uint32_t v, float s) {
    return pack_bf16x2(bf16lo(v) * s, bf16hi(v) * s);
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
__device__ __forceinline__ bool warp_wait_b(uint64_t* bar, uint32_t parity, const Abort& ab) {
    const bool r = mbar_wait(bar, parity, ab);
    return __all_sync(0xffffffffu, r);
}
__device__ __forceinline__ void drain(uint64_t* bar, uint32_t parity, uint64_t ns) {
    const uint64_t t0 = globaltimer();
    while (!mbar_try_wait(bar, parity) && globaltimer() - t0 < ns) {
    }
}

// K-major SW128 operand (rows of 64 elements, 128 B), K step kk of 16 elements; 64-element
// K atoms are rows * 128 B apart.
__device__ __forceinline__ uint64_t bdesc_k(uint32_t base, int kk, int rows) {
    return sdesc_sw128(base + (uint32_t)(kk >> 2) * rows * 128u + (uint32_t)(kk & 3) * 32u, 16u,
                       1024u);
}
// MN-major SW128 operand (each 128 B row holds 64 MN elements of one K index), K step kk of
// 16 rows; 64-element MN atoms are `lbo` bytes apart.
__device__ __forceinline__ uint64_t bdesc_mn(uint32_t base, int kk, uint32_t lbo) {
    return sdesc_sw128(base + (uint32_t)kk * 2048u, lbo, 1024u);
}
// byte offset of element (row, col) in a tile of `rows` rows whose columns come in 64-wide
// SW128 atoms placed rows * 128 B apart
__device__ __forceinline__ uint32_t tile_off(int row, int col, int rows) {
    return (uint32_t)(col >> 6) * rows * 128u + sw128_off(row, col & 63);
}

// Per-token coefficients of tokens [t0, t0 + Q) of (b, h), by one warp, into shared arrays.
// Tokens past T have dt = A = lam = 0 (no decay, no input).  u = Q is the next chunk's first
// token (its dt and lam give the last token's trapezoid share).
struct Coefs {
    float* dd;    // dt          [Q + 1]
    float* ll;    // lam         [Q + 1]
    float* aa;    // A           [Q]
    float* cr;    // chunk-relative inclusive prefix of dt A   [Q]
    float* gam;   // lam dt      [Q]
    float* nx;    // (1 - lam_{u+1}) dt_{u+1}   [Q]
    float* ew;    // e_u w_u     [Q]
    float* ee;    // e_u = e^{cr_{Q-1} - cr_u}  [Q]
    float* ff;    // f_u = e^{cr_u}             [Q]
    __device__ explicit Coefs(float* base) {
        dd = base;
        ll = dd + kQ + 1;
        aa = ll + kQ + 1;
        cr = aa + kQ;
        gam = cr + kQ;
        nx = gam + kQ;
        ew = nx + kQ;
        ee = ew + kQ;
        ff = ee + kQ;
    }
    static constexpr int kFloats = 2 * (kQ + 1) + 7 * kQ;
};

// Per-token coefficients of a chunk of QT tokens (QT = 64 / R), one warp, two tokens a lane.
// Slots u >= QT hold zeros, except that slot QT holds the next token's dt and lam.
template <int QT>
__device__ void chunk_coefs(const BwdArgs& a, int b, int h, long long t0, const Coefs& k) {
    const int lane = threadIdx.x & 31;
    const long long T = a.T;
    float d2[2], l2[2], a2[2];
    // with QT = 64 the next token has no slot of its own: lane 0 requests it with its tokens
    float dn = 0.f, ln = 0.f;
    if (QT == kQ && lane == 0 && t0 + kQ < T) {
        const size_t o = ((size_t)b * T + t0 + kQ) * a.H + h;
        dn = a.dt[o];
        ln = a.lam[o];
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int u = 2 * lane + i;
        const long long t = t0 + u;
        const bool ok = u <= QT && t < T;
        const size_t o = ((size_t)b * T + (ok ? t : 0)) * a.H + h;
        d2[i] = ok ? a.dt[o] : 0.f;
        l2[i] = ok ? a.lam[o] : 0.f;
        a2[i] = ok && u < QT ? a.A[o] : 0.f;
    }
    const float e0 = d2[0] * a2[0], e1 = d2[1] * a2[1];
    float s = e0 + e1;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float v = __shfl_up_sync(0xffffffffu, s, o);
        if (lane >= o) s += v;
    }
    const float cend = __shfl_sync(0xffffffffu, s, 31);
    const float c0 = (s - (e0 + e1)) + e0, c1 = c0 + e1;
    const float cc[2] = {c0, c1};
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int u = 2 * lane + i;
        const bool in = u < QT;
        k.dd[u] = d2[i];
        k.ll[u] = l2[i];
        k.aa[u] = a2[i];
        k.cr[u] = in ? cc[i] : 0.f;
        k.gam[u] = in ? l2[i] * d2[i] : 0.f;
        k.ee[u] = in ? ex2f((cend - cc[i]) * kLog2e) : 0.f;
        k.ff[u] = in ? ex2f(cc[i] * kLog2e) : 0.f;
    }
    if (QT == kQ && lane == 0) {
        k.dd[kQ] = dn;
        k.ll[kQ] = ln;
    }
    __syncwarp();
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int u = 2 * lane + i;
        const float nx = u < QT ? (1.f - k.ll[u + 1]) * k.dd[u + 1] : 0.f;
        k.nx[u] = nx;
        k.ew[u] = k.ee[u] * (k.gam[u] + nx);
    }
    __syncwarp();
}

// ------------------------------------------------------------------------------------
// 1. chunk products
template <int NST>
struct VuCfg {
    static constexpr int NT = 256;                           // threads
    static constexpr int NH = NST / 2;
    static constexpr int OFF_B = 0;                          // B~ [NST/64][Q][64] bf16
    static constexpr int OFF_C = kQ * NST * 2;               // C~
    static constexpr int OFF_XW = 2 * kQ * NST * 2;          // diag(e w) X [Q][64]
    static constexpr int OFF_DYF = OFF_XW + kQ * kPc * 2;    // diag(f) dY [Q][64]
    static constexpr int OFF_COEF = OFF_DYF + kQ * kPc * 2;
    static constexpr int OFF_SEG = OFF_COEF + Coefs::kFloats * 4;   // [NT / NH][NH] angle sums
    static constexpr int OFF_BAR = (OFF_SEG + NT * 4 + 7) / 8 * 8;
    static constexpr int OFF_MISC = OFF_BAR + 8;
    static constexpr int USED = OFF_MISC + 16 + 1024;
    // at least 50 KB, so that at most four CTAs (4 x 128 TMEM columns) share an SM
    static constexpr int SMEM = USED > 51200 ? USED : 51200;
    static constexpr uint32_t ID = idesc_bf16(NST, kPc, true, true);
    static_assert(SMEM * 5 > 233472 && SMEM * 4 <= 233472 - 4096, "at most four CTAs per SM");
};

// 256 threads: thread (pair j, row segment sg) holds TPS = 64 / (256 / NH) tile rows of one
// pair (TPS / R tokens), so that every global input of the chunk (X and dY rows, the angles,
// the B and C pairs) is requested in one round before the first barrier.  A tile row is one
// (token, rank): row = R u + r.
template <int NST, int RK>
__global__ void __launch_bounds__(256, 2) bwd_vu_kernel(const __grid_constant__ TcBwd p) {
    using C = VuCfg<NST>;
    constexpr int NH = C::NH, QT = kQ / RK;
    const BwdArgs& a = p.a;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + C::OFF_BAR);
    uint32_t* misc = reinterpret_cast<uint32_t*>(sm + C::OFF_MISC);
    const Coefs k(reinterpret_cast<float*>(sm + C::OFF_COEF));
    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    const int c = (int)(blockIdx.x % p.nch);
    const size_t bh = blockIdx.x / p.nch;
    const int b = (int)(bh / a.H), h = (int)(bh % a.H), g = h / (a.H / a.G);
    const long long t0 = (long long)c * QT;
    const size_t cc = bh * p.nch + c;

    constexpr int SEGS = C::NT / NH, TPS = kQ / SEGS, TT = TPS / RK, XT = 2 * kQ * 8 / C::NT;
    static_assert(TT * RK == TPS, "a segment holds whole tokens");
    const int j = tid % NH, sg = tid / NH;
    const bool angle = (a.flags & M3_FLAG_THETA_IS_ANGLE) != 0;
    uint4 xv[XT];
    float thv[TT];
    uint32_t pbv[TPS], pcv[TPS];
    {
        const uint16_t* xg = static_cast<const uint16_t*>(a.x);
        const uint16_t* yg = static_cast<const uint16_t*>(a.dy);
        const uint16_t* Bg = static_cast<const uint16_t*>(a.B);
        const uint16_t* Cg = static_cast<const uint16_t*>(a.C);
#pragma unroll
        for (int m = 0; m < XT; ++m) {
            const int i = tid + C::NT * m;
            const bool isY = i >= kQ * 8;
            const int e = isY ? i - kQ * 8 : i;
            const int row = e >> 3;
            const long long t = t0 + row / RK;
            xv[m] = t < a.T ? *reinterpret_cast<const uint4*>(
                                  (isY ? yg : xg) +
                                  ((((size_t)b * a.T + t) * a.H + h) * RK + row % RK) * kPc + (e & 7) * 8)
                            : make_uint4(0u, 0u, 0u, 0u);
        }
        // row sg TPS + i holds rank i % R of token (sg TPS + i) / R (TPS is a multiple of R);
        // a token's angle is loaded with its first rank's B and C pair
#pragma unroll
        for (int i = 0; i < TPS; ++i) {
            const long long t = t0 + (sg * TPS + i) / RK;
            if (i % RK == 0) thv[i / RK] = 0.f;
            pbv[i] = pcv[i] = 0u;
            if (t < a.T) {
                const size_t tr = ((size_t)b * a.T + t) * a.G + g;
                if (i % RK == 0) thv[i / RK] = a.theta[tr * NH + j];
                const size_t o = (tr * RK + i % RK) * NST + 2 * j;
                pbv[i] = *reinterpret_cast<const uint32_t*>(Bg + o);
                pcv[i] = *reinterpret_cast<const uint32_t*>(Cg + o);
            }
        }
    }
    if (tid == 0) {
        mbar_init(&bar[0], 1);
        misc[1] = 0u;
        fence_mbar_init();
    }
    if (w == 1) {
        tmem_alloc(&misc[0], 128);
        tmem_relinquish();
    }
    if (w == 0) chunk_coefs<QT>(a, b, h, t0, k);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc[0];
    const Abort ab{reinterpret_cast<volatile uint32_t*>(&misc[1]), p.status, p.limit_ns};
    if (tid == 0) p.ctot[cc] = k.cr[QT - 1];

    // diag(e w) X and diag(f) dY
#pragma unroll
    for (int m = 0; m < XT; ++m) {
        const int i = tid + C::NT * m;
        const bool isY = i >= kQ * 8;
        const int e = isY ? i - kQ * 8 : i;
        const int row = e >> 3;
        const float sc = isY ? k.ff[row / RK] : k.ew[row / RK];
        const uint4 v = xv[m];
        *reinterpret_cast<uint4*>(sm + (isY ? C::OFF_DYF : C::OFF_XW) + sw128_off(row, (e & 7) * 8)) =
            make_uint4(scale2(v.x, sc), scale2(v.y, sc), scale2(v.z, sc), scale2(v.w, sc));
    }
    // B~, C~ in the chunk's frame: the segment's angle sums, the segments' totals exchanged,
    // then the rotation of the segment's tokens
    {
        float* segt = reinterpret_cast<float*>(sm + C::OFF_SEG);
        float rho[TT];
        float r = 0.f;
#pragma unroll
        for (int i = 0; i < TT; ++i) {
            r += angle ? thv[i] : k.dd[sg * TT + i] * thv[i];
            rho[i] = r;
        }
        segt[sg * NH + j] = r;
        __syncthreads();
        float off = 0.f;
        for (int s2 = 0; s2 < sg; ++s2) off += segt[s2 * NH + j];
        if (sg == SEGS - 1) p.atot[cc * NH + j] = off + r;
#pragma unroll
        for (int i = 0; i < TPS; ++i) {
            const int u = sg * TPS + i;   // tile row
            float sn, cs;
            __sincosf(wrap_angle(off + rho[i / RK]), &sn, &cs);
            const float b0 = bf16lo(pbv[i]), b1 = bf16hi(pbv[i]), c0 = bf16lo(pcv[i]), c1 = bf16hi(pcv[i]);
            const uint32_t o = tile_off(u, 2 * j, kQ);
            *reinterpret_cast<uint32_t*>(sm + C::OFF_B + o) =
                pack_bf16x2(fmaf(cs, b0, sn * b1), fmaf(cs, b1, -sn * b0));
            *reinterpret_cast<uint32_t*>(sm + C::OFF_C + o) =
                pack_bf16x2(fmaf(cs, c0, sn * c1), fmaf(cs, c1, -sn * c0));
        }
    }
    fence_proxy_async_smem();
    __syncthreads();

    if (tid == 0) {
        tc_fence_after();
        const uint32_t sb = smem_u32(sm);
#pragma unroll
        for (int kk = 0; kk < kQ / 16; ++kk)
            mma_bf16(tmem, bdesc_mn(sb + C::OFF_B, kk, kQ * 128), bdesc_mn(sb + C::OFF_XW, kk, kQ * 128),
                     C::ID, kk > 0);
#pragma unroll
        for (int kk = 0; kk < kQ / 16; ++kk)
            mma_bf16(tmem + 64, bdesc_mn(sb + C::OFF_C, kk, kQ * 128),
                     bdesc_mn(sb + C::OFF_DYF, kk, kQ * 128), C::ID, kk > 0);
        mma_commit(&bar[0]);
    }
    const bool ok = warp_wait_b(&bar[0], 0, ab);
    tc_fence_after();
    if (ok) {
        // warps 0-3 read V (columns 0-63), warps 4-7 read U (columns 64-127)
        const int q = w & 3, m = w >> 2;
        const uint32_t tq = tmem + ((uint32_t)(32 * q) << 16);
        uint16_t* dst0 = (m ? p.U : p.V) + cc * (size_t)NST * kPc;
#pragma unroll
        for (int cb = 0; cb < 32; cb += 16) {
            uint32_t r[16], r2[16];
            int n, col, col2;
            if constexpr (NST == 128) {   // M = 128: row = lane of the quadrant
                tmem_ld_32x32b_x16(tq + 64 * m + 2 * cb, r);
                tmem_ld_32x32b_x16(tq + 64 * m + 2 * cb + 16, r2);
                n = 32 * q + lane;
                col = 2 * cb;
                col2 = 2 * cb + 16;
            } else {                      // M = 64: 16 rows per quadrant, column halves
                tmem_ld_16x32bx2_x16<32>(tq + 64 * m + cb, r);
                n = 16 * q + (lane & 15);
                col = cb + 32 * (lane >> 4);
                col2 = -1;
            }
            tmem_wait_ld();
            uint4* d = reinterpret_cast<uint4*>(dst0 + (size_t)n * kPc + col);
#pragma unroll
            for (int i = 0; i < 2; ++i)
                d[i] = make_uint4(pack_bf16x2(__uint_as_float(r[8 * i]), __uint_as_float(r[8 * i + 1])),
                                  pack_bf16x2(__uint_as_float(r[8 * i + 2]), __uint_as_float(r[8 * i + 3])),
                                  pack_bf16x2(__uint_as_float(r[8 * i + 4]), __uint_as_float(r[8 * i + 5])),
                                  pack_bf16x2(__uint_as_float(r[8 * i + 6]), __uint_as_float(r[8 * i + 7])));
            if (col2 >= 0) {
                uint4* d2 = reinterpret_cast<uint4*>(dst0 + (size_t)n * kPc + col2);
#pragma unroll
                for (int i = 0; i < 2; ++i)
                    d2[i] = make_uint4(pack_bf16x2(__uint_as_float(r2[8 * i]), __uint_as_float(r2[8 * i + 1])),
                                       pack_bf16x2(__uint_as_float(r2[8 * i + 2]), __uint_as_float(r2[8 * i + 3])),
                                       pack_bf16x2(__uint_as_float(r2[8 * i + 4]), __uint_as_float(r2[8 * i + 5])),
                                       pack_bf16x2(__uint_as_float(r2[8 * i + 6]), __uint_as_float(r2[8 * i + 7])));
            }
        }
    }
    if (tid == 0 && !ok) drain(&bar[0], 0, 100000000ull);
    tc_fence_before();
    __syncthreads();
    if (w == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, 128);
    }
}

// ------------------------------------------------------------------------------------
// 2. chunk scan: thread (channel p, pair group pg) holds state rows 2j, 2j+1 of column p for
// the pairs j = pg + NPG k, k < 8.  A chunk's inputs (its V or U tile, the stored entering
// state, the angles and the decay) come through a ring of SCAN_KS shared-memory stages
// filled by cp.async SCAN_KS - 1 chunks ahead, every thread copying 16-byte pieces.
__device__ __forceinline__ void cpa16(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cpa4(void* dst, const void* src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cpa_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cpa_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory"); }

constexpr int SCAN_KS = 3;
template <int NST>
struct ScanCfg {
    static constexpr int TILE = NST * kPc * 2;                 // one [N][P] bf16 tile
    static constexpr int VEC = NST / 2 * 4;                    // one fp32 value per pair
    static constexpr int STAGE = 2 * TILE + VEC + 16;          // tile, tile, pairs, decay
    static constexpr int SMEM = SCAN_KS * STAGE;
};

template <int NST, int RK>
__global__ void __launch_bounds__(4 * NST, NST == 128 ? 1 : 2) bwd_scan_kernel(const __grid_constant__ TcBwd p) {
    constexpr int NH = NST / 2, NPG = NST / 16, NT = 4 * NST, NW = NT / 32;
    using SC = ScanCfg<NST>;
    const BwdArgs& a = p.a;
    extern __shared__ __align__(128) uint8_t ring[];
    __shared__ float red[2][NW];
    __shared__ float part[RK][NPG][kPc];
    __shared__ float exs[NH];
    const int tid = threadIdx.x, pc = tid & 63, pg = tid >> 6, lane = tid & 31, w = tid >> 5;
    const size_t bh = blockIdx.x;
    const int b = (int)(bh / a.H), h = (int)(bh % a.H), g = h / (a.H / a.G);
    const int nch = p.nch;
    const size_t NP = (size_t)NST * kPc;
    if (tid < NH) exs[tid] = 0.f;
    __syncthreads();

    // starting state g0 = h0 + (1 - lam_0) dt_0 sum_r B_prev,r x_prev,r^T
    const size_t o0 = (size_t)b * a.T * a.H + h;
    const float k0 = (1.f - a.lam[o0]) * a.dt[o0];
    float xp[RK];
#pragma unroll
    for (int r = 0; r < RK; ++r) xp[r] = bf_at(a.x_prev, (bh * RK + r) * kPc + pc);
    const size_t bprow = ((size_t)b * a.G + g) * RK * NST;   // B_prev row of rank r: + r NST
    float ge[8], go[8], P[8];
#pragma unroll
    for (int kx = 0; kx < 8; ++kx) {
        const int j = pg + NPG * kx;
        float se = 0.f, so = 0.f;
#pragma unroll
        for (int r = 0; r < RK; ++r) {
            se = fmaf(bf_at(a.B_prev, bprow + r * NST + 2 * j), xp[r], se);
            so = fmaf(bf_at(a.B_prev, bprow + r * NST + 2 * j + 1), xp[r], so);
        }
        ge[kx] = fmaf(k0, se, a.h0[bh * NP + (size_t)(2 * j) * kPc + pc]);
        go[kx] = fmaf(k0, so, a.h0[bh * NP + (size_t)(2 * j + 1) * kPc + pc]);
        P[kx] = 0.f;
    }
    // forward: the state entering every chunk, then the chunk's contribution in the call
    // frame; stage c % KS holds chunk c's V tile, angles and decay
    auto issue_fwd = [&](int c) {
        const size_t cc = bh * nch + c;
        uint8_t* d = ring + (c % SCAN_KS) * SC::STAGE;
        const uint8_t* V = reinterpret_cast<const uint8_t*>(p.V + cc * NP);
        for (int i = tid; i < SC::TILE / 16; i += NT) cpa16(d + 16 * i, V + 16 * i);
        if (tid < SC::VEC / 16) cpa16(d + 2 * SC::TILE + 16 * tid, p.atot + cc * NH + 4 * tid);
        if (tid == NT - 1) cpa4(d + 2 * SC::TILE + SC::VEC, p.ctot + cc);
    };
#pragma unroll
    for (int i = 0; i < SCAN_KS - 1; ++i) {
        if (i < nch) issue_fwd(i);
        cpa_commit();
    }
    for (int c = 0; c < nch; ++c) {
        const size_t cc = bh * nch + c;
        cpa_wait<SCAN_KS - 2>();   // this thread's copies of chunk c have landed
        // one barrier: chunk c's stage is complete, and every thread is done with the stage of
        // chunk c - 1, which the next copies refill
        __syncthreads();
        if (c + SCAN_KS - 1 < nch) issue_fwd(c + SCAN_KS - 1);
        cpa_commit();
        const uint8_t* st = ring + (c % SCAN_KS) * SC::STAGE;
        const uint16_t* vt = reinterpret_cast<const uint16_t*>(st);
        const float* at = reinterpret_cast<const float*>(st + 2 * SC::TILE);
        const float dec = ex2f(at[NH] * kLog2e);
        uint8_t* gt = reinterpret_cast<uint8_t*>(p.gin) + cc * NP * 2;
#pragma unroll
        for (int kx = 0; kx < 8; ++kx) {
            const int j = pg + NPG * kx;
            if (pc == 0) p.P0[(bh * (nch + 1) + c) * NH + j] = P[kx];
            *reinterpret_cast<uint16_t*>(gt + sw128_off(2 * j, pc)) = to_bf(ge[kx]);
            *reinterpret_cast<uint16_t*>(gt + sw128_off(2 * j + 1, pc)) = to_bf(go[kx]);
            const float v0 = __uint_as_float((uint32_t)vt[(2 * j) * kPc + pc] << 16);
            const float v1 = __uint_as_float((uint32_t)vt[(2 * j + 1) * kPc + pc] << 16);
            float sn, cs;
            __sincosf(P[kx], &sn, &cs);
            ge[kx] = fmaf(dec, ge[kx], fmaf(cs, v0, sn * v1));
            go[kx] = fmaf(dec, go[kx], fmaf(cs, v1, -sn * v0));
            P[kx] = wrap_angle(P[kx] + at[j]);
        }
    }
    // the final state and dL/dh_T: dg = R(-psi_T) dH; the last token's angle gradient
    // sum_p dH_odd (R(psi_T) g)_even - dH_even (R(psi_T) g)_odd
    float de[8], dq[8];
#pragma unroll
    for (int kx = 0; kx < 8; ++kx) {
        const int j = pg + NPG * kx;
        if (pc == 0) p.P0[(bh * (nch + 1) + nch) * NH + j] = P[kx];
        de[kx] = 0.f;
        dq[kx] = 0.f;
        if (a.dhT) {
            float sn, cs;
            __sincosf(P[kx], &sn, &cs);
            const float d0 = a.dhT[bh * NP + (size_t)(2 * j) * kPc + pc];
            const float d1 = a.dhT[bh * NP + (size_t)(2 * j + 1) * kPc + pc];
            de[kx] = fmaf(cs, d0, sn * d1);
            dq[kx] = fmaf(cs, d1, -sn * d0);
            const float h0 = fmaf(cs, ge[kx], -sn * go[kx]), h1 = fmaf(sn, ge[kx], cs * go[kx]);
            const float ex = warp_sum(fmaf(d1, h0, -d0 * h1));
            if (lane == 0) atomicAdd(&exs[j], ex);
        }
    }
    __syncthreads();   // the chunk-start angles (global) and exs are complete
    if (tid < NH) p.extra[bh * NH + tid] = exs[tid];
    // reverse: the adjoint of the state leaving every chunk; stage i % KS (i = nch - 1 - c)
    // holds chunk c's U tile, its stored entering state, the angles before it and its decay.
    // The entering states and angles were written by this CTA's forward sweep (ordered before
    // these copies by the barrier above).
    auto issue_rev = [&](int i) {
        const int c = nch - 1 - i;
        const size_t cc = bh * nch + c;
        uint8_t* d = ring + (i % SCAN_KS) * SC::STAGE;
        const uint8_t* Uc = reinterpret_cast<const uint8_t*>(p.U + cc * NP);
        const uint8_t* gt = reinterpret_cast<const uint8_t*>(p.gin) + cc * NP * 2;
        for (int e = tid; e < SC::TILE / 16; e += NT) {
            cpa16(d + 16 * e, Uc + 16 * e);
            cpa16(d + SC::TILE + 16 * e, gt + 16 * e);
        }
        if (tid < SC::VEC / 16)
            cpa16(d + 2 * SC::TILE + 16 * tid, p.P0 + (bh * (nch + 1) + c) * NH + 4 * tid);
        if (tid == NT - 1) cpa4(d + 2 * SC::TILE + SC::VEC, p.ctot + cc);
    };
    __syncthreads();   // every thread is past its last read of the forward stages
#pragma unroll
    for (int i = 0; i < SCAN_KS - 1; ++i) {
        if (i < nch) issue_rev(i);
        cpa_commit();
    }
    // q of chunk c: the warps' partial sums in red[c & 1], added by thread 0 behind the next
    // barrier (the next step writes the other half)
    float dec_prev = 0.f;
    auto finish_q = [&](int c) {
        float t = 0.f;
        for (int k = 0; k < NW; ++k) t += red[c & 1][k];
        p.q[bh * nch + c] = dec_prev * t;
    };
    for (int i = 0; i < nch; ++i) {
        const int c = nch - 1 - i;
        const size_t cc = bh * nch + c;
        cpa_wait<SCAN_KS - 2>();   // this thread's copies of chunk c have landed
        // one barrier: chunk c's stage is complete, every thread is done with the stage of
        // step i - 1 (refilled next), and the partial sums of chunk c + 1 are in red
        __syncthreads();
        if (tid == 0 && i > 0) finish_q(c + 1);
        if (i + SCAN_KS - 1 < nch) issue_rev(i + SCAN_KS - 1);
        cpa_commit();
        const uint8_t* st = ring + (i % SCAN_KS) * SC::STAGE;
        const uint16_t* ut = reinterpret_cast<const uint16_t*>(st);
        const uint8_t* gs = st + SC::TILE;
        const float* pt = reinterpret_cast<const float*>(st + 2 * SC::TILE);
        const float dec = ex2f(pt[NH] * kLog2e);
        uint8_t* dt_ = reinterpret_cast<uint8_t*>(p.dgo) + cc * NP * 2;
        float s = 0.f;
#pragma unroll
        for (int kx = 0; kx < 8; ++kx) {
            const int j = pg + NPG * kx;
            *reinterpret_cast<uint16_t*>(dt_ + sw128_off(2 * j, pc)) = to_bf(de[kx]);
            *reinterpret_cast<uint16_t*>(dt_ + sw128_off(2 * j + 1, pc)) = to_bf(dq[kx]);
            const float g0 = __uint_as_float((uint32_t)*reinterpret_cast<const uint16_t*>(gs + sw128_off(2 * j, pc)) << 16);
            const float g1 = __uint_as_float((uint32_t)*reinterpret_cast<const uint16_t*>(gs + sw128_off(2 * j + 1, pc)) << 16);
            s = fmaf(de[kx], g0, fmaf(dq[kx], g1, s));
            const float u0 = __uint_as_float((uint32_t)ut[(2 * j) * kPc + pc] << 16);
            const float u1 = __uint_as_float((uint32_t)ut[(2 * j + 1) * kPc + pc] << 16);
            float sn, cs;
            __sincosf(pt[j], &sn, &cs);
            de[kx] = fmaf(dec, de[kx], fmaf(cs, u0, sn * u1));
            dq[kx] = fmaf(dec, dq[kx], fmaf(cs, u1, -sn * u0));
        }
        s = warp_sum(s);
        if (lane == 0) red[c & 1][w] = s;
        dec_prev = dec;
    }
    __syncthreads();
    if (tid == 0) finish_q(0);   // before the starting-state sums below reuse red[0]
    // the starting state: dh0 = dg; dx_prev,r = k0 B_prev,r^T dg; dB_prev,r += k0 dg x_prev,r;
    // v0 = sum_r <dg, B_prev,r x_prev,r^T> (for dt_0 and lam_0)
    float pp[RK];
#pragma unroll
    for (int r = 0; r < RK; ++r) pp[r] = 0.f;
#pragma unroll
    for (int kx = 0; kx < 8; ++kx) {
        const int j = pg + NPG * kx;
        a.dh0[bh * NP + (size_t)(2 * j) * kPc + pc] = de[kx];
        a.dh0[bh * NP + (size_t)(2 * j + 1) * kPc + pc] = dq[kx];
#pragma unroll
        for (int r = 0; r < RK; ++r) {
            const size_t br = bprow + r * NST + 2 * j;
            pp[r] = fmaf(de[kx], bf_at(a.B_prev, br), fmaf(dq[kx], bf_at(a.B_prev, br + 1), pp[r]));
            const float se = warp_sum(de[kx] * xp[r]), so = warp_sum(dq[kx] * xp[r]);
            if (lane == 0) {
                atomicAdd(a.dB_prev + br, k0 * se);
                atomicAdd(a.dB_prev + br + 1, k0 * so);
            }
        }
    }
    float sv = 0.f;
#pragma unroll
    for (int r = 0; r < RK; ++r) {
        part[r][pg][pc] = pp[r];
        sv = fmaf(pp[r], xp[r], sv);
    }
    sv = warp_sum(sv);
    __syncthreads();
    if (lane == 0) red[0][w] = sv;
    for (int e = tid; e < RK * kPc; e += NT) {
        const int r = e / kPc, c2 = e % kPc;
        float t = 0.f;
        for (int i = 0; i < NPG; ++i) t += part[r][i][c2];
        a.dx_prev[(bh * RK + r) * kPc + c2] = k0 * t;
    }
    __syncthreads();
    if (tid == 0) {
        float t = 0.f;
        for (int i = 0; i < NW; ++i) t += red[0][i];
        p.v0[bh] = t;
    }
}

// ------------------------------------------------------------------------------------
// 3. chunk gradients
//
// Two CTAs share an SM: each allocates 256 TMEM columns after its loads, and keeps under
// 113 KB of shared memory.  TMEM: columns [0, 64) hold S, then B~ dg, then dX; [64, 128)
// dY X^T; [128, 128 + N) dY g^T, then dC~, then dB~.  Three MMA rounds:
//   1. S = C~ B~^T, dY X^T, dY g^T;            epilogue: L o S, dS, the band and decay sums,
//                                              <C~_t, (dY g^T)_t>, row scale f
//   2. dC~ += dS B~, B~ dg;                    epilogue: dC~ rotated back (dC), angle terms;
//                                              <X_s, (B~ dg)_s>, row scale e w; X <- e w X
//   3. dX = (L o S)^T dY + ., dB~ = (e w X) dg^T + dS^T C~;   epilogue: dX, dB
// Tile rows are (token, rank) pairs, 64 / R tokens of R ranks: the masks and scales are the
// row's token's, and the per-token sums (band weights, log-decay, angles) gather its R rows.
template <int NST, int RK>
struct GrCfg {
    static constexpr int NH = NST / 2;
    static constexpr int T64 = kQ * 128;                      // one [Q][64] bf16 tile
    static constexpr int OFF_X = 0, OFF_DY = T64, OFF_MS = 2 * T64, OFF_DS = 3 * T64;
    static constexpr int OFF_C = 4 * T64;                     // C~ [NST/64][Q][64]
    static constexpr int OFF_B = OFF_C + kQ * NST * 2;        // B~
    static constexpr int OFF_GIN = OFF_B + kQ * NST * 2;      // g_in [NST][64]
    static constexpr int OFF_DG = OFF_GIN + NST * kPc * 2;    // dg_out [NST][64]
    static constexpr int OFF_SEG = OFF_DG + NST * kPc * 2;    // fp32 [256 / NH][NH]
    static constexpr int OFF_COEF = OFF_SEG + 256 * 4;
    static constexpr int NACC = 10;
    static constexpr int OFF_ACC = OFF_COEF + Coefs::kFloats * 4;
    static constexpr int OFF_BAR = (OFF_ACC + (NACC * kQ + 4) * 4 + 7) / 8 * 8;
    static constexpr int OFF_MISC = OFF_BAR + 4 * 8;
    // with R > 1 the R rows of a token add their angle gradients into a table of their own
    // [Q / R][NH] fp32 (the angle table is still read while they are formed)
    static constexpr int OFF_DPS = OFF_MISC + 16;
    static constexpr int USED = OFF_DPS + (RK > 1 ? (kQ / RK) * NH * 4 : 0) + 1024;
    // two CTAs per SM (2 x 256 TMEM columns), never three
    static constexpr int SMEM = USED > 79872 ? USED : 79872;
    static_assert(2 * (SMEM + 1024) <= 233472 && 3 * (SMEM + 1024) > 233472, "two CTAs per SM");
    // the angle table [Q][NH] fp32 lives in the L o S / dS tiles until the first epilogue and
    // in the g_in tile after it (both free at those times)
    static_assert(kQ * NH * 4 <= 2 * T64 && kQ * NH * 4 <= NST * kPc * 2, "angle table");
    static constexpr uint32_t TM_A = 0, TM_GX = 64, TM_C = 128;
    static constexpr uint32_t ID_QQ = idesc_bf16(kQ, kQ, false, false);    // S, dY X^T
    static constexpr uint32_t ID_BDG = idesc_bf16(kQ, kPc, false, true);   // B~ dg
    static constexpr uint32_t ID_KN = idesc_bf16(kQ, NST, false, false);   // dY g^T, X dg^T
    static constexpr uint32_t ID_MSDY = idesc_bf16(kQ, kPc, true, true);   // (L o S)^T dY
    static constexpr uint32_t ID_DSB = idesc_bf16(kQ, NST, false, true);   // dS B~
    static constexpr uint32_t ID_DSC = idesc_bf16(kQ, NST, true, true);    // dS^T C~
};

// angle table index: row u, pair j, XOR-swizzled so that a column read by the 16 rows of a
// half warp hits 16 banks
template <int NH>
__device__ __forceinline__ int psi_idx(int u, int j) {
    return u * NH + (j ^ (u & 31));
}

// TMEM access of an M = 64 accumulator by 8 warps: warp w reaches lane quadrant w % 4 (rows
// 16 q .. 16 q + 15 at lanes 32 q .. 32 q + 15); 16-column blocks cb of the first half go to
// warp group w / 4 in turn; a thread's lane half (lane / 16) takes block cb + NC / 2.
template <int NC>
__device__ __forceinline__ void ld_blk(uint32_t tq, uint32_t col, int cb, uint32_t (&r)[16]) {
    tmem_ld_16x32bx2_x16<NC / 2>(tq + col + cb, r);
}
template <int NC>
__device__ __forceinline__ void st_blk(uint32_t tq, uint32_t col, int cb, const uint32_t (&r)[16]) {
    tmem_st_16x32bx2_x16<NC / 2>(tq + col + cb, r);
}

// sum over the 16 lanes of a half warp of 16 per-lane column values: lane l ends with the
// sum of column l % 16 (recursive halving: 15 shuffles)
__device__ __forceinline__ float colsum16(float (&v)[16], int lane) {
#pragma unroll
    for (int o = 8; o >= 1; o >>= 1) {
        const bool up = (lane & o) != 0;
#pragma unroll
        for (int i = 0; i < o; ++i) {
            const float send = up ? v[i] : v[i + o];
            const float keep = up ? v[i + o] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
    }
    return v[0];
}

template <int NST, int RK>
__global__ void __launch_bounds__(256, 2) bwd_grads_kernel(const __grid_constant__ TcBwd p) {
    using C = GrCfg<NST, RK>;
    constexpr int NH = C::NH, QT = kQ / RK;
    const BwdArgs& a = p.a;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + C::OFF_BAR);
    uint32_t* misc = reinterpret_cast<uint32_t*>(sm + C::OFF_MISC);
    const Coefs k(reinterpret_cast<float*>(sm + C::OFF_COEF));
    float* acc = reinterpret_cast<float*>(sm + C::OFF_ACC);
    float* rs = acc;              // row sums of dL om E
    float* cs = acc + kQ;         // column sums of dL om E
    float* ga = acc + 2 * kQ;     // column sums of dL E over t >= s
    float* dgd = acc + 3 * kQ;    // diagonal dL E
    float* dv = acc + 4 * kQ;     // <X_s, (B~ dg)_s>
    float* qz = acc + 5 * kQ;     // <C~_t, (dY g^T)_t>
    float* dcm = acc + 6 * kQ;    // log-decay gradient, then its suffix sums
    float* dnx = acc + 7 * kQ;    // band-weight gradient owed to the next token
    float* misc2 = acc + 9 * kQ;  // [0] dD partial, [1..2] warp sums, [3] suffix carry
    float* psi0 = reinterpret_cast<float*>(sm + C::OFF_MS);    // angle table, first home
    float* psi1 = reinterpret_cast<float*>(sm + C::OFF_GIN);   // and second
    float* dpsi = RK > 1 ? reinterpret_cast<float*>(sm + C::OFF_DPS) : psi1;   // angle gradients
    float* segt = reinterpret_cast<float*>(sm + C::OFF_SEG);
    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    const int c = (int)(blockIdx.x % p.nch);
    const size_t bh = blockIdx.x / p.nch;
    const int b = (int)(bh / a.H), h = (int)(bh % a.H), g = h / (a.H / a.G);
    const long long t0 = (long long)c * QT;
    const int nv = (int)(a.T - t0 < QT ? a.T - t0 : QT);   // tokens of the chunk
    const size_t cc = bh * p.nch + c;
    const bool angle = (a.flags & M3_FLAG_THETA_IS_ANGLE) != 0;
    const uint32_t tile_bytes = NST * kPc * 2;

    if (tid == 0) {
        for (int i = 0; i < 4; ++i) mbar_init(&bar[i], 1);
        misc[1] = 0u;
        fence_mbar_init();
        mbar_arrive_expect_tx(&bar[0], 2 * tile_bytes);
        bulk_load(sm + C::OFF_GIN, reinterpret_cast<const uint8_t*>(p.gin) + cc * tile_bytes,
                  tile_bytes, &bar[0]);
        bulk_load(sm + C::OFF_DG, reinterpret_cast<const uint8_t*>(p.dgo) + cc * tile_bytes,
                  tile_bytes, &bar[0]);
    }
    if (w == 1) chunk_coefs<QT>(a, b, h, t0, k);
    for (int i = tid; i < C::NACC * kQ + 4; i += 256) acc[i] = 0.f;
    if constexpr (RK > 1)
        for (int i = tid; i < QT * NH; i += 256) dpsi[i] = 0.f;
    // Every global input of the chunk is requested before any of it is used: the angle
    // prefix's theta and dt, the chunk-start angle, the X and dY rows, and the B and C pairs
    // of the rotation (with N = 128 those follow once the angle prefix has consumed theta and
    // dt, to keep the registers in flight under the budget of two CTAs).
    constexpr int SEGS = 256 / NH, TPS = QT / SEGS;   // tokens of a (pair, segment)
    static_assert(TPS * SEGS == QT, "whole tokens per segment");
    const int jj = tid % NH, sg = tid / NH;
    // B~, C~ in the call frame: thread (pair jr, tile rows ur + RS m) for m < KT
    constexpr int KT = kQ * NH / 256, RS = 256 / NH;
    constexpr bool BC_EARLY = NST == 64;
    const int jr = tid % NH, ur = tid / NH;
    uint32_t pbv[KT], pcv[KT];
    auto load_bc = [&]() {
        const uint16_t* Bg = static_cast<const uint16_t*>(a.B);
        const uint16_t* Cg = static_cast<const uint16_t*>(a.C);
#pragma unroll
        for (int m = 0; m < KT; ++m) {
            const int rw = ur + RS * m;
            const long long t = t0 + rw / RK;
            pbv[m] = pcv[m] = 0u;
            if (t < a.T) {
                const size_t o = ((((size_t)b * a.T + t) * a.G + g) * RK + rw % RK) * NST + 2 * jr;
                pbv[m] = *reinterpret_cast<const uint32_t*>(Bg + o);
                pcv[m] = *reinterpret_cast<const uint32_t*>(Cg + o);
            }
        }
    };
    const float p0 = p.P0[(bh * (p.nch + 1) + c) * NH + jj];
    if constexpr (BC_EARLY) load_bc();
    float rho[TPS];
    {
        float thv[TPS], dtv[TPS];
#pragma unroll
        for (int i = 0; i < TPS; ++i) {
            const long long t = t0 + sg * TPS + i;
            const bool in = t < a.T;
            const size_t bt = (size_t)b * a.T + (in ? t : 0);
            thv[i] = in ? a.theta[(bt * a.G + g) * NH + jj] : 0.f;
            dtv[i] = in ? a.dt[bt * a.H + h] : 0.f;
        }
        constexpr int XT = 2 * kQ * 8 / 256;   // X / dY 16-byte pieces per thread
        uint4 xv[XT];
        const uint16_t* xg = static_cast<const uint16_t*>(a.x);
        const uint16_t* yg = static_cast<const uint16_t*>(a.dy);
#pragma unroll
        for (int m = 0; m < XT; ++m) {
            const int i = tid + 256 * m;
            const bool isY = i >= kQ * 8;
            const int e = isY ? i - kQ * 8 : i;
            const int row = e >> 3;
            const long long t = t0 + row / RK;
            xv[m] = t < a.T ? *reinterpret_cast<const uint4*>(
                                  (isY ? yg : xg) +
                                  ((((size_t)b * a.T + t) * a.H + h) * RK + row % RK) * kPc + (e & 7) * 8)
                            : make_uint4(0u, 0u, 0u, 0u);
        }
        float r = 0.f;
#pragma unroll
        for (int i = 0; i < TPS; ++i) {
            r += angle ? thv[i] : dtv[i] * thv[i];
            rho[i] = r;
        }
        segt[sg * NH + jj] = r;
        // theta and dt are consumed: their registers take the B and C pairs
        if constexpr (!BC_EARLY) load_bc();
#pragma unroll
        for (int m = 0; m < XT; ++m) {
            const int i = tid + 256 * m;
            const bool isY = i >= kQ * 8;
            const int e = isY ? i - kQ * 8 : i;
            *reinterpret_cast<uint4*>(sm + (isY ? C::OFF_DY : C::OFF_X) + sw128_off(e >> 3, (e & 7) * 8)) = xv[m];
        }
    }
    __syncthreads();
    {
        float off = p0;
        for (int s2 = 0; s2 < sg; ++s2) off += segt[s2 * NH + jj];
#pragma unroll
        for (int i = 0; i < TPS; ++i) psi0[psi_idx<NH>(sg * TPS + i, jj)] = wrap_angle(off + rho[i]);
    }
    __syncthreads();
#pragma unroll
    for (int m = 0; m < KT; ++m) {
        const int u = ur + RS * m;   // tile row
        float sn, cs2;
        __sincosf(psi0[psi_idx<NH>(u / RK, jr)], &sn, &cs2);
        const float b0 = bf16lo(pbv[m]), b1 = bf16hi(pbv[m]), c0 = bf16lo(pcv[m]), c1 = bf16hi(pcv[m]);
        const uint32_t off = tile_off(u, 2 * jr, kQ);
        *reinterpret_cast<uint32_t*>(sm + C::OFF_B + off) =
            pack_bf16x2(fmaf(cs2, b0, sn * b1), fmaf(cs2, b1, -sn * b0));
        *reinterpret_cast<uint32_t*>(sm + C::OFF_C + off) =
            pack_bf16x2(fmaf(cs2, c0, sn * c1), fmaf(cs2, c1, -sn * c0));
    }
    fence_proxy_async_smem();
    if (w == 0) {
        tmem_alloc(&misc[0], 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc[0];
    const Abort ab{reinterpret_cast<volatile uint32_t*>(&misc[1]), p.status, p.limit_ns};
    const uint32_t sb = smem_u32(sm);
    int issued = 0;   // thread 0: MMA rounds issued
    if (tid == 0) {
        // test hook of the failure path: a wait that nothing completes (bar[3] only follows
        // round 3) gives up after the call's limit, raising the abort flag and the status
        const bool stall = (a.flags & M3_FLAG_TEST_STALL) != 0;
        if (stall) (void)mbar_wait(&bar[3], 0, ab);
        if (!stall && mbar_wait(&bar[0], 0, ab)) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < NST / 16; ++kk)
                mma_bf16(tmem + C::TM_A, bdesc_k(sb + C::OFF_C, kk, kQ), bdesc_k(sb + C::OFF_B, kk, kQ),
                         C::ID_QQ, kk > 0);
#pragma unroll
            for (int kk = 0; kk < kPc / 16; ++kk)
                mma_bf16(tmem + C::TM_GX, bdesc_k(sb + C::OFF_DY, kk, kQ), bdesc_k(sb + C::OFF_X, kk, kQ),
                         C::ID_QQ, kk > 0);
#pragma unroll
            for (int kk = 0; kk < kPc / 16; ++kk)
                mma_bf16(tmem + C::TM_C, bdesc_k(sb + C::OFF_DY, kk, kQ),
                         bdesc_k(sb + C::OFF_GIN, kk, NST), C::ID_KN, kk > 0);
            mma_commit(&bar[1]);
            issued = 1;
        } else {
            drain(&bar[0], 0, 100000000ull);   // let the copies land before the CTA exits
        }
    }

    const int q4 = w & 3, wg = w >> 2, hf = lane >> 4;
    const int t = 16 * q4 + (lane & 15);          // this thread's accumulator row
    const int tu = t / RK;                        // and its token
    const uint32_t tq = tmem + ((uint32_t)(32 * q4) << 16);
    auto flag_ok = [&]() { return *reinterpret_cast<volatile uint32_t*>(&misc[1]) == 0u; };

    // ---- first epilogue: masks, band and decay sums, <C~_t, (dY g^T)_t>, row scale f
    bool ok = warp_wait_b(&bar[1], 0, ab);
    tc_fence_after();
    if (ok) {   // the angle table moves to the g_in tile (read by round 1, now free)
        constexpr int CP = kQ * NH * 4 / 16 / 256;
        const uint4* src = reinterpret_cast<const uint4*>(psi0);
        uint4* dst = reinterpret_cast<uint4*>(psi1);
#pragma unroll
        for (int i = 0; i < CP; ++i) dst[tid + 256 * i] = src[tid + 256 * i];
    }
    __syncthreads();
    ok = ok && flag_ok();
    if (ok) {
        const float crt = k.cr[tu];
        {
            const int cb = 16 * wg, col0 = cb + 32 * hf;
            uint32_t sv[16], gv[16];
            ld_blk<64>(tq, C::TM_A, cb, sv);
            ld_blk<64>(tq, C::TM_GX, cb, gv);
            tmem_wait_ld();
            float ca[16], cbv[16], rsum = 0.f, ddiag = 0.f, dgl = 0.f;
            bool dgh = false;
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                uint32_t ms[4], ds[4];
#pragma unroll
                for (int i2 = 0; i2 < 8; i2 += 2) {
                    float mv[2], dvv[2];
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int i = 8 * hh + i2 + e;
                        const int s = col0 + i, su = s / RK;
                        const bool in = su <= tu;
                        const float E = in ? ex2f((crt - k.cr[su]) * kLog2e) : 0.f;
                        const float om = in ? k.gam[su] + (su < tu ? k.nx[su] : 0.f) : 0.f;
                        const float L = E * om;
                        const float S = __uint_as_float(sv[i]), G = __uint_as_float(gv[i]);
                        mv[e] = S * L;
                        dvv[e] = G * L;
                        const float dom = S * G * E;
                        ca[i] = dom * om;
                        cbv[i] = dom;
                        rsum += dom * om;
                        if (su == tu) {
                            dgl += dom;
                            dgh = true;
                        }
                        if (s == t) ddiag = G;
                    }
                    ms[i2 / 2] = pack_bf16x2(mv[0], mv[1]);
                    ds[i2 / 2] = pack_bf16x2(dvv[0], dvv[1]);
                }
                *reinterpret_cast<uint4*>(sm + C::OFF_MS + sw128_off(t, col0 + 8 * hh)) =
                    make_uint4(ms[0], ms[1], ms[2], ms[3]);
                *reinterpret_cast<uint4*>(sm + C::OFF_DS + sw128_off(t, col0 + 8 * hh)) =
                    make_uint4(ds[0], ds[1], ds[2], ds[3]);
            }
            if (ddiag != 0.f) atomicAdd(&misc2[0], ddiag);
            if (dgh) atomicAdd(&dgd[tu], dgl);
            const float csum = colsum16(ca, lane), gsum = colsum16(cbv, lane);
            atomicAdd(&cs[(col0 + (lane & 15)) / RK], csum);
            atomicAdd(&ga[(col0 + (lane & 15)) / RK], gsum);
            rsum += __shfl_xor_sync(0xffffffffu, rsum, 16);
            if (hf == 0) atomicAdd(&rs[tu], rsum);
        }
        {
            float d = 0.f;
            const float sf = k.ff[tu];
#pragma unroll
            for (int m = 0; m < NST / 64; ++m) {
                const int cb = 16 * (wg + 2 * m), col0 = cb + (NST / 2) * hf;
                uint32_t v[16];
                ld_blk<NST>(tq, C::TM_C, cb, v);
                tmem_wait_ld();
                const uint4 c0 = *reinterpret_cast<const uint4*>(sm + C::OFF_C + tile_off(t, col0, kQ));
                const uint4 c1 = *reinterpret_cast<const uint4*>(sm + C::OFF_C + tile_off(t, col0 + 8, kQ));
                const uint32_t ct[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float a0 = __uint_as_float(v[2 * i]), a1 = __uint_as_float(v[2 * i + 1]);
                    d = fmaf(bf16lo(ct[i]), a0, fmaf(bf16hi(ct[i]), a1, d));
                    v[2 * i] = __float_as_uint(a0 * sf);
                    v[2 * i + 1] = __float_as_uint(a1 * sf);
                }
                st_blk<NST>(tq, C::TM_C, cb, v);
            }
            d += __shfl_xor_sync(0xffffffffu, d, 16);
            if (hf == 0) atomicAdd(&qz[tu], d);
        }
        tmem_wait_st();
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    ok = ok && flag_ok();
    if (tid == 0 && issued == 1) {
        if (ok) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < kQ / 16; ++kk)
                mma_bf16(tmem + C::TM_C, bdesc_k(sb + C::OFF_DS, kk, kQ),
                         bdesc_mn(sb + C::OFF_B, kk, kQ * 128), C::ID_DSB, 1);
#pragma unroll
            for (int kk = 0; kk < NST / 16; ++kk)
                mma_bf16(tmem + C::TM_A, bdesc_k(sb + C::OFF_B, kk, kQ),
                         bdesc_mn(sb + C::OFF_DG, kk, tile_bytes), C::ID_BDG, kk > 0);
            mma_commit(&bar[2]);
            issued = 2;
        } else {
            drain(&bar[1], 0, 100000000ull);
        }
    }

    // ---- second epilogue: <X_s, (B~ dg)_s>, row scale e w, X <- e w X; dC~ rotated back
    const long long tg = t0 + tu;
    const bool live = tu < nv;
    const size_t grow = ((((size_t)b * a.T + (live ? tg : 0)) * a.G + g) * RK + t % RK) * NST;
    constexpr int NB = NST / 64;          // 16-column blocks per thread in an N-wide tile
    float dps[NB * 8];                    // this thread's angle gradients (from dC~)
    ok = ok && warp_wait_b(&bar[2], 0, ab);
    tc_fence_after();
    if (ok) {
        {
            const int cb = 16 * wg, col0 = cb + 32 * hf;
            uint32_t v[16];
            ld_blk<64>(tq, C::TM_A, cb, v);
            tmem_wait_ld();
            uint4* xp0 = reinterpret_cast<uint4*>(sm + C::OFF_X + sw128_off(t, col0));
            uint4* xp1 = reinterpret_cast<uint4*>(sm + C::OFF_X + sw128_off(t, col0 + 8));
            const uint4 x0 = *xp0, x1 = *xp1;
            const uint32_t xs[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
            float d = 0.f;
            const float sc = k.ew[tu];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float a0 = __uint_as_float(v[2 * i]), a1 = __uint_as_float(v[2 * i + 1]);
                d = fmaf(bf16lo(xs[i]), a0, fmaf(bf16hi(xs[i]), a1, d));
                v[2 * i] = __float_as_uint(a0 * sc);
                v[2 * i + 1] = __float_as_uint(a1 * sc);
            }
            st_blk<64>(tq, C::TM_A, cb, v);
            *xp0 = make_uint4(scale2(x0.x, sc), scale2(x0.y, sc), scale2(x0.z, sc), scale2(x0.w, sc));
            *xp1 = make_uint4(scale2(x1.x, sc), scale2(x1.y, sc), scale2(x1.z, sc), scale2(x1.w, sc));
            d += __shfl_xor_sync(0xffffffffu, d, 16);
            if (hf == 0) atomicAdd(&dv[tu], d);
        }
        const uint16_t* Cg = static_cast<const uint16_t*>(a.C);
#pragma unroll
        for (int m = 0; m < NB; ++m) {
            const int cb = 16 * (wg + 2 * m), col0 = cb + (NST / 2) * hf;
            uint4 rc[2] = {make_uint4(0u, 0u, 0u, 0u), make_uint4(0u, 0u, 0u, 0u)};
            if (live) {
                rc[0] = *reinterpret_cast<const uint4*>(Cg + grow + col0);
                rc[1] = *reinterpret_cast<const uint4*>(Cg + grow + col0 + 8);
            }
            uint32_t vc[16];
            ld_blk<NST>(tq, C::TM_C, cb, vc);
            tmem_wait_ld();
            const uint32_t cw[8] = {rc[0].x, rc[0].y, rc[0].z, rc[0].w, rc[1].x, rc[1].y, rc[1].z, rc[1].w};
            float oc[16];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                float sn, cs2;
                __sincosf(psi1[psi_idx<NH>(tu, col0 / 2 + i)], &sn, &cs2);
                const float c0 = bf16lo(cw[i]), c1 = bf16hi(cw[i]);
                const float ct0 = fmaf(cs2, c0, sn * c1), ct1 = fmaf(cs2, c1, -sn * c0);
                const float dc0 = __uint_as_float(vc[2 * i]), dc1 = __uint_as_float(vc[2 * i + 1]);
                dps[8 * m + i] = fmaf(dc0, ct1, -dc1 * ct0);
                oc[2 * i] = fmaf(cs2, dc0, -sn * dc1);
                oc[2 * i + 1] = fmaf(sn, dc0, cs2 * dc1);
            }
            if (live) {
                float4* dC = reinterpret_cast<float4*>(a.dC + grow + col0);
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    atomicAdd(dC + i, make_float4(oc[4 * i], oc[4 * i + 1], oc[4 * i + 2], oc[4 * i + 3]));
            }
        }
        tmem_wait_st();
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    ok = ok && flag_ok();
    if (tid == 0 && issued == 2) {
        if (ok) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < kQ / 16; ++kk)
                mma_bf16(tmem + C::TM_A, bdesc_mn(sb + C::OFF_MS, kk, kQ * 128),
                         bdesc_mn(sb + C::OFF_DY, kk, kQ * 128), C::ID_MSDY, 1);
#pragma unroll
            for (int kk = 0; kk < kPc / 16; ++kk)
                mma_bf16(tmem + C::TM_C, bdesc_k(sb + C::OFF_X, kk, kQ),
                         bdesc_k(sb + C::OFF_DG, kk, NST), C::ID_KN, kk > 0);
#pragma unroll
            for (int kk = 0; kk < kQ / 16; ++kk)
                mma_bf16(tmem + C::TM_C, bdesc_mn(sb + C::OFF_DS, kk, kQ * 128),
                         bdesc_mn(sb + C::OFF_C, kk, kQ * 128), C::ID_DSC, 1);
            mma_commit(&bar[3]);
            issued = 3;
        } else {
            drain(&bar[2], 0, 100000000ull);
        }
    }

    // ---- third epilogue: dX; dB~ rotated back; the angle gradient of every (token, pair)
    ok = ok && warp_wait_b(&bar[3], 0, ab);
    tc_fence_after();
    if (ok) {
        {
            const int cb = 16 * wg, col0 = cb + 32 * hf;
            uint32_t v[16];
            ld_blk<64>(tq, C::TM_A, cb, v);
            tmem_wait_ld();
            const float Dh = a.D ? a.D[h] : 0.f;
            const uint4 y0 = *reinterpret_cast<const uint4*>(sm + C::OFF_DY + sw128_off(t, col0));
            const uint4 y1 = *reinterpret_cast<const uint4*>(sm + C::OFF_DY + sw128_off(t, col0 + 8));
            const uint32_t ys[8] = {y0.x, y0.y, y0.z, y0.w, y1.x, y1.y, y1.z, y1.w};
            if (live) {
                float4* dst = reinterpret_cast<float4*>(
                    a.dx + ((((size_t)b * a.T + tg) * a.H + h) * RK + t % RK) * kPc + col0);
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    dst[i] = make_float4(fmaf(Dh, bf16lo(ys[2 * i]), __uint_as_float(v[4 * i])),
                                         fmaf(Dh, bf16hi(ys[2 * i]), __uint_as_float(v[4 * i + 1])),
                                         fmaf(Dh, bf16lo(ys[2 * i + 1]), __uint_as_float(v[4 * i + 2])),
                                         fmaf(Dh, bf16hi(ys[2 * i + 1]), __uint_as_float(v[4 * i + 3])));
            }
        }
        const uint16_t* Bg = static_cast<const uint16_t*>(a.B);
#pragma unroll
        for (int m = 0; m < NB; ++m) {
            const int cb = 16 * (wg + 2 * m), col0 = cb + (NST / 2) * hf;
            uint4 rb[2] = {make_uint4(0u, 0u, 0u, 0u), make_uint4(0u, 0u, 0u, 0u)};
            if (live) {
                rb[0] = *reinterpret_cast<const uint4*>(Bg + grow + col0);
                rb[1] = *reinterpret_cast<const uint4*>(Bg + grow + col0 + 8);
            }
            uint32_t vb[16];
            ld_blk<NST>(tq, C::TM_C, cb, vb);
            tmem_wait_ld();
            const uint32_t bw[8] = {rb[0].x, rb[0].y, rb[0].z, rb[0].w, rb[1].x, rb[1].y, rb[1].z, rb[1].w};
            float ob[16];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int j = col0 / 2 + i;
                float sn, cs2;
                __sincosf(psi1[psi_idx<NH>(tu, j)], &sn, &cs2);
                const float b0 = bf16lo(bw[i]), b1 = bf16hi(bw[i]);
                const float bt0 = fmaf(cs2, b0, sn * b1), bt1 = fmaf(cs2, b1, -sn * b0);
                const float db0 = __uint_as_float(vb[2 * i]), db1 = __uint_as_float(vb[2 * i + 1]);
                const float gp = dps[8 * m + i] + fmaf(db0, bt1, -db1 * bt0);
                if constexpr (RK == 1)
                    psi1[psi_idx<NH>(t, j)] = gp;   // the angle is read by this thread alone
                else
                    atomicAdd(&dpsi[psi_idx<NH>(tu, j)], gp);
                ob[2 * i] = fmaf(cs2, db0, -sn * db1);
                ob[2 * i + 1] = fmaf(sn, db0, cs2 * db1);
            }
            if (live) {
                float4* dB = reinterpret_cast<float4*>(a.dB + grow + col0);
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    atomicAdd(dB + i, make_float4(ob[4 * i], ob[4 * i + 1], ob[4 * i + 2], ob[4 * i + 3]));
            }
        }
    }
    // TMEM is no longer read: release it for the SM's other CTA
    if (tid == 0 && issued > 0) drain(&bar[issued], 0, 100000000ull);
    tc_fence_before();
    __syncthreads();
    if (w == 0) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
    ok = ok && flag_ok();

    // angles: suffix sums over the chunk's tokens per (pair, token segment), then the
    // segments' totals; each head's chunk-local sums go to the workspace, where the finish
    // step adds the carry from later chunks and sums over the group's heads
    float loc[TPS];
    if (ok) {
        float r = 0.f;
#pragma unroll
        for (int i = TPS - 1; i >= 0; --i) {
            r += dpsi[psi_idx<NH>(sg * TPS + i, jj)];
            loc[i] = r;
        }
        segt[sg * NH + jj] = r;
        // the log-decay gradient of every token (chunk-local: its terms sum to zero over the
        // chunk, so the suffix sums that reach dA and dt stay inside the chunk)
        if (tid < kQ) {
            const int u = tid;
            const float ewdv = k.ew[u] * dv[u];
            dcm[u] = rs[u] - cs[u] + k.ff[u] * qz[u] - ewdv;
            const float sw = warp_sum(ewdv);
            if (lane == 0) misc2[1 + w] = sw;
            const float dw = k.ee[u] * dv[u];
            dnx[u] = ga[u] - dgd[u] + dw;
        }
    }
    __syncthreads();
    if (ok) {
        float off = 0.f;
        for (int s2 = sg + 1; s2 < SEGS; ++s2) off += segt[s2 * NH + jj];
        float* pg = p.pang + (bh * a.T + t0) * NH + jj;
#pragma unroll
        for (int i = 0; i < TPS; ++i) {
            const int u = sg * TPS + i;
            if (u < nv) pg[(size_t)u * NH] = loc[i] + off;
        }
        if (sg == 0) p.dtot[cc * NH + jj] = loc[0] + off;
    }
    if (ok && tid < kQ) {
        const int u = tid;
        float v = dcm[u];
        if (u == nv - 1) v += misc2[1] + misc2[2] + p.q[cc];
        // suffix sum over u within the warp, then warp 0 adds warp 1's total
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float x = __shfl_down_sync(0xffffffffu, v, o);
            if (lane + o < 32) v += x;
        }
        const float w1 = __shfl_sync(0xffffffffu, v, 0);
        if (w == 1 && lane == 0) misc2[3] = w1;
        __syncwarp();
        dcm[u] = v;
    }
    __syncthreads();
    if (ok && tid < kQ) {
        const int u = tid;
        const float dda = dcm[u] + (w == 0 ? misc2[3] : 0.f);
        const float dga = k.ee[u] * dv[u] + ga[u];
        float ddt = fmaf(dda, k.aa[u], dga * k.ll[u]);
        float dlam = dga * k.dd[u];
        if (u > 0) {
            ddt = fmaf(dnx[u - 1], 1.f - k.ll[u], ddt);
            dlam = fmaf(-dnx[u - 1], k.dd[u], dlam);
        }
        if (c == 0 && u == 0) {
            const float v0 = p.v0[bh];
            ddt = fmaf(1.f - k.ll[0], v0, ddt);
            dlam = fmaf(-k.dd[0], v0, dlam);
        }
        if (u < nv) {
            const size_t o = ((size_t)b * a.T + t0 + u) * a.H + h;
            a.ddt[o] = ddt;
            a.dA[o] = dda * k.dd[u];
            a.dlam[o] = dlam;
        }
        if (u == QT - 1) p.spill[cc] = dnx[u];
        if (u == 0 && a.D && a.dD) atomicAdd(&a.dD[h], misc2[0]);
    }
}

// ------------------------------------------------------------------------------------
// 4. finish.  The carry of every chunk: carry[c] = extra + sum over later chunks of their
// angle-gradient totals (a suffix sum over chunks, one thread per (batch, head, pair)).
__global__ void bwd_carry_kernel(const __grid_constant__ TcBwd p, int NH) {
    const long long n = (long long)p.a.batch * p.a.H * NH;
    const long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x;
    if (e >= n) return;
    const long long bh = e / NH;
    const int j = (int)(e % NH);
    float run = p.extra[e];
    for (int c = p.nch - 1; c >= 0; --c) {
        const size_t o = ((size_t)bh * p.nch + c) * NH + j;
        p.carry[o] = run;
        run += p.dtot[o];
    }
}

// Per (batch, chunk, group): dtheta of every token = sum over the group's heads of the full
// angle gradient (chunk-local sums plus carry) times dt (1 with the angle flag), in a fixed
// order; dt of every (token, head) gets the full angle gradient . theta, and the chunk's
// first token the previous chunk's last-token share of the trapezoid weight.  Heads go in
// tiles of 64: thread (token u, pair quarter jq) accumulates dtheta over the tile's heads
// (read-only loads only) and leaves each head's theta product in shared memory; then every
// (token, head) of the tile updates its dt and lam.
template <int NH>
__global__ void __launch_bounds__(256, 2) bwd_finish_kernel(const __grid_constant__ TcBwd p) {
    constexpr int JP = NH / 4, HT = 64;
    const BwdArgs& a = p.a;
    __shared__ float sdt[kQ][HT + 1];
    const int tid = threadIdx.x, u = tid >> 2, jq = tid & 3;
    const int c = (int)(blockIdx.x % p.nch);
    const long long bg = blockIdx.x / p.nch;
    const int g = (int)(bg % a.G), b = (int)(bg / a.G);
    const int hpg = a.H / a.G;
    const long long t0 = (long long)c * p.qt, t = t0 + u;
    const int nv = (int)(a.T - t0 < p.qt ? a.T - t0 : p.qt);
    const bool live = u < nv;
    const bool angle = (a.flags & M3_FLAG_THETA_IS_ANGLE) != 0;
    const size_t trow = ((size_t)b * a.T + (live ? t : 0)) * a.G + g;
    float th[JP], acc[JP];
#pragma unroll
    for (int i = 0; i < JP; ++i) {
        th[i] = (live && !angle) ? a.theta[trow * NH + jq * JP + i] : 0.f;
        acc[i] = 0.f;
    }
    for (int h0 = 0; h0 < hpg; h0 += HT) {
        const int nh = hpg - h0 < HT ? hpg - h0 : HT;
#pragma unroll 4
        for (int hh = 0; hh < nh; ++hh) {
            const int h = g * hpg + h0 + hh;
            const size_t bh = (size_t)b * a.H + h;
            const float* pg = p.pang + (bh * a.T + (live ? t : 0)) * NH + jq * JP;
            const float* cg = p.carry + (bh * p.nch + c) * NH + jq * JP;
            const float d = live ? __ldg(a.dt + ((size_t)b * a.T + (live ? t : 0)) * a.H + h) : 0.f;
            float s = 0.f;
#pragma unroll
            for (int i4 = 0; i4 < JP / 4; ++i4) {
                float4 pv = make_float4(0.f, 0.f, 0.f, 0.f), cv = pv;
                if (live) {
                    pv = __ldg(reinterpret_cast<const float4*>(pg) + i4);
                    cv = __ldg(reinterpret_cast<const float4*>(cg) + i4);
                }
                const float dv[4] = {pv.x + cv.x, pv.y + cv.y, pv.z + cv.z, pv.w + cv.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int i = 4 * i4 + e;
                    acc[i] = fmaf(dv[e], angle ? 1.f : d, acc[i]);
                    s = fmaf(dv[e], th[i], s);
                }
            }
            s += __shfl_xor_sync(0xffffffffu, s, 1);
            s += __shfl_xor_sync(0xffffffffu, s, 2);
            if (jq == 0) sdt[u][hh] = s;
        }
        __syncthreads();
        // dt and lam of the tile's (token, head) pairs: 16 per thread, loads before stores
        constexpr int PER = kQ * HT / 256;
        float cur[PER];
#pragma unroll
        for (int m = 0; m < PER; ++m) {
            const int e = tid + 256 * m, uu = e / HT, hh = e % HT;
            cur[m] = (uu < nv && hh < nh) ? a.ddt[((size_t)b * a.T + t0 + uu) * a.H + g * hpg + h0 + hh] : 0.f;
        }
#pragma unroll
        for (int m = 0; m < PER; ++m) {
            const int e = tid + 256 * m, uu = e / HT, hh = e % HT;
            if (uu >= nv || hh >= nh) continue;
            const int h = g * hpg + h0 + hh;
            const size_t o = ((size_t)b * a.T + t0 + uu) * a.H + h;
            float add = sdt[uu][hh];
            if (uu == 0 && c > 0) {
                const float sp = p.spill[((size_t)b * a.H + h) * p.nch + c - 1];
                add = fmaf(sp, 1.f - a.lam[o], add);
                a.dlam[o] -= sp * a.dt[o];
            }
            a.ddt[o] = cur[m] + add;
        }
        __syncthreads();
    }
    if (live) {
#pragma unroll
        for (int i = 0; i < JP; ++i) a.dtheta[trow * NH + jq * JP + i] = acc[i];
    }
}

struct Layout {
    size_t V, U, gin, dgo, ctot, atot, P0, q, dtot, spill, extra, v0, pang, carry, bytes;
};

Layout layout(int batch, int H, int N, int R, long long T) {
    const long long qt = kQ / R;
    const size_t BH = (size_t)batch * H, nch = (size_t)((T + qt - 1) / qt), NP = (size_t)N * kPc;
    const size_t NH = N / 2;
    Layout L;
    size_t o = 0;
    auto take = [&](size_t bytes) {
        const size_t at = o;
        o += (bytes + 255) / 256 * 256;
        return at;
    };
    L.V = take(BH * nch * NP * 2);
    L.U = take(BH * nch * NP * 2);
    L.gin = take(BH * nch * NP * 2);
    L.dgo = take(BH * nch * NP * 2);
    L.ctot = take(BH * nch * 4);
    L.atot = take(BH * nch * NH * 4);
    L.P0 = take(BH * (nch + 1) * NH * 4);
    L.q = take(BH * nch * 4);
    L.dtot = take(BH * nch * NH * 4);
    L.spill = take(BH * nch * 4);
    L.extra = take(BH * NH * 4);
    L.v0 = take(BH * 4);
    L.pang = take(BH * (size_t)T * NH * 4);
    L.carry = take(BH * nch * NH * 4);
    L.bytes = o;
    return L;
}

template <int NST, int RK>
cudaError_t launch_n(const TcBwd& p, long long units, cudaStream_t s) {
    const int smv = VuCfg<NST>::SMEM, smg = GrCfg<NST, RK>::SMEM;
    cudaError_t e = cudaFuncSetAttribute(bwd_vu_kernel<NST, RK>, cudaFuncAttributeMaxDynamicSharedMemorySize, smv);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(bwd_grads_kernel<NST, RK>, cudaFuncAttributeMaxDynamicSharedMemorySize, smg);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(bwd_scan_kernel<NST, RK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             ScanCfg<NST>::SMEM);
    if (e != cudaSuccess) return e;
    bwd_vu_kernel<NST, RK><<<(unsigned)units, VuCfg<NST>::NT, smv, s>>>(p);
    bwd_scan_kernel<NST, RK><<<(unsigned)((size_t)p.a.batch * p.a.H), 4 * NST, ScanCfg<NST>::SMEM, s>>>(p);
    bwd_grads_kernel<NST, RK><<<(unsigned)units, 256, smg, s>>>(p);
    const long long bhj = (long long)p.a.batch * p.a.H * (NST / 2);
    bwd_carry_kernel<<<(unsigned)((bhj + 255) / 256), 256, 0, s>>>(p, NST / 2);
    bwd_finish_kernel<NST / 2><<<(unsigned)((long long)p.a.batch * p.a.G * p.nch), 256, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace

bool scan_bwd_tc_ok(int io_dtype, int N, int P, int R) {
    return io_dtype == M3_BF16 && P == kPc &&
           ((R == 1 && (N == 64 || N == 128)) || ((R == 2 || R == 4) && N == 64));
}

size_t scan_bwd_tc_workspace_bytes(int batch, int H, int N, int R, long long T) {
    return layout(batch, H, N, R, T).bytes;
}

cudaError_t launch_scan_bwd_tc(const BwdArgs& a, int R, void* ws, uint32_t* status,
                               unsigned long long limit_ns, cudaStream_t s) {
    const Layout L = layout(a.batch, a.H, a.N, R, a.T);
    uint8_t* base = static_cast<uint8_t*>(ws);
    TcBwd p;
    p.a = a;
    p.qt = kQ / R;
    p.nch = (int)((a.T + p.qt - 1) / p.qt);
    p.V = reinterpret_cast<uint16_t*>(base + L.V);
    p.U = reinterpret_cast<uint16_t*>(base + L.U);
    p.gin = reinterpret_cast<uint16_t*>(base + L.gin);
    p.dgo = reinterpret_cast<uint16_t*>(base + L.dgo);
    p.ctot = reinterpret_cast<float*>(base + L.ctot);
    p.atot = reinterpret_cast<float*>(base + L.atot);
    p.P0 = reinterpret_cast<float*>(base + L.P0);
    p.q = reinterpret_cast<float*>(base + L.q);
    p.dtot = reinterpret_cast<float*>(base + L.dtot);
    p.spill = reinterpret_cast<float*>(base + L.spill);
    p.extra = reinterpret_cast<float*>(base + L.extra);
    p.v0 = reinterpret_cast<float*>(base + L.v0);
    p.pang = reinterpret_cast<float*>(base + L.pang);
    p.carry = reinterpret_cast<float*>(base + L.carry);
    p.status = status;
    p.limit_ns = limit_ns;
    const long long units = (long long)a.batch * a.H * p.nch;
    if (a.N == 128) return launch_n<128, 1>(p, units, s);
    if (R == 2) return launch_n<64, 2>(p, units, s);
    if (R == 4) return launch_n<64, 4>(p, units, s);
    return launch_n<64, 1>(p, units, s);
}

}  // namespace m3
