"""Pure-Python brute force of the SVDQuant layer, for tiny shapes only.

Written independently of ``oracle/`` (no NumPy arithmetic, exact rational
nearest-value searches, struct-based float32 rounding, frexp-based bfloat16
rounding) so that it can pin the oracle: a plausible slip in the oracle
(a dropped term, a swapped operand, a wrong rounding) shows up as a mismatch.
"""

import math
import struct
from fractions import Fraction


def f32r(x):
    """Round a Python float to the nearest float32 (ties to even)."""
    return struct.unpack("<f", struct.pack("<f", x))[0]


def f16r(x):
    """Round to the nearest IEEE half (ties to even, subnormals kept), saturating at 65504."""
    if x == 0.0:
        return x
    a = min(abs(x), 65504.0)
    m, e = math.frexp(a)              # a = m 2^e, m in [0.5, 1)
    q = 2.0 ** max(e - 11, -24)       # 11 significant bits; subnormal quantum 2^-24
    r = round(a / q) * q              # Python round: ties to even
    r = min(r, 65504.0)
    return math.copysign(r, x)


def bf16r(x):
    """Round to 8 significant bits, ties to even (normal range)."""
    if x == 0.0:
        return x
    m, e = math.frexp(x)
    return math.ldexp(round(m * 256.0), e - 8)


def _table(kind):
    out = []
    if kind == "e2m1":
        for code in range(8):
            e, m = code >> 1, code & 1
            v = Fraction(m, 2) if e == 0 else Fraction(2) ** (e - 1) * (1 + Fraction(m, 2))
            out.append((v, code))
    else:
        for code in range(127):
            e, m = code >> 3, code & 7
            v = Fraction(m, 512) if e == 0 else Fraction(2) ** (e - 7) * (1 + Fraction(m, 8))
            out.append((v, code))
    return out


E2M1 = _table("e2m1")
E4M3 = _table("e4m3")


def nearest(x, table, sign_bit):
    """Nearest table value by exact rational distance, ties to the even code."""
    a = abs(Fraction(x))
    best = None
    for v, code in table:
        d = abs(a - v)
        if best is None or d < best[0] or (d == best[0] and code % 2 == 0):
            best = (d, code)
    code = best[1]
    if math.copysign(1.0, x) < 0:
        code |= sign_bit
    return code


def value(code, table, sign_bit):
    v = float(table[code & ~sign_bit][0])
    return -v if code & sign_bit else v


def quantize_block(block, g):
    """Two-level NVFP4 quantization of 16 float32 values with tensor scale g."""
    amax = max(abs(t) for t in block)
    c = f32r(1.0 / f32r(6.0 * g))
    s = nearest(f32r(amax * c), E4M3, 0x80)
    d = f32r(value(s, E4M3, 0x80) * g)
    rcp = 0.0 if d == 0.0 else f32r(1.0 / d)
    codes = [nearest(f32r(t * rcp), E2M1, 0x8) for t in block]
    return codes, s


def global_scale(amax):
    return 1.0 if amax == 0.0 else f32r(amax / 2688.0)


def quantize_rows(rows, g):
    codes, scales = [], []
    for row in rows:
        rc, rs = [], []
        for b in range(0, len(row), 16):
            c, s = quantize_block(row[b:b + 16], g)
            rc += c
            rs.append(s)
        codes.append(rc)
        scales.append(rs)
    return codes, scales


def deq(codes, scales):
    return [[value(c, E2M1, 0x8) * value(scales[i][k // 16], E4M3, 0x80) for k, c in enumerate(row)]
            for i, row in enumerate(codes)]


def layer_forward(W, X, act_amax, L1, L2, bias=None, gelu=False):
    """Whole layer on nested lists: W [N][K], X [M][K], L1 [K][r], L2 [r][N]."""
    N, K = len(W), len(W[0])
    M = len(X)
    r = len(L2)
    w_amax = [max(abs(W[n][j]) for n in range(N)) for j in range(K)]
    lam, inv = [], []
    for j in range(K):
        a, w = act_amax[j], w_amax[j]
        lj = 1.0 if (a == 0.0 or w == 0.0) else f32r(math.sqrt(f32r(a / w)))
        lam.append(lj)
        inv.append(f32r(1.0 / lj))
    # residual of the smoothed weight, rank-one terms in order
    R = [[lam[j] * W[n][j] for n in range(N)] for j in range(K)]
    for i in range(r):
        for j in range(K):
            for n in range(N):
                R[j][n] = R[j][n] - L1[j][i] * L2[i][n]
    R32t = [[f32r(R[j][n]) for j in range(K)] for n in range(N)]
    g_w = global_scale(max(abs(v) for row in R32t for v in row))
    wc, ws = quantize_rows(R32t, g_w)
    xh = [[bf16r(f32r(X[m][j] * inv[j])) for j in range(K)] for m in range(M)]
    g_a = global_scale(max(bf16r(f32r(act_amax[j] * inv[j])) for j in range(K)))
    ac, as_ = quantize_rows(xh, g_a)
    da, dw = deq(ac, as_), deq(wc, ws)
    lr = [[sum(xh[m][j] * L1[j][i] for j in range(K)) for i in range(r)] for m in range(M)]
    Y = []
    for m in range(M):
        row = []
        for n in range(N):
            y = g_a * g_w * sum(da[m][k] * dw[n][k] for k in range(K))
            y += sum(lr[m][i] * L2[i][n] for i in range(r))
            if bias is not None:
                y += bias[n]
            if gelu:
                y = 0.5 * y * (1.0 + math.tanh(math.sqrt(2.0 / math.pi) * (y + 0.044715 * y ** 3)))
            row.append(y)
        Y.append(row)
    return dict(lam=lam, inv=inv, g_w=g_w, g_a=g_a, w_codes=wc, w_scales=ws, a_codes=ac,
                a_scales=as_, x_hat=xh, lr=lr, Y=Y)


def qkv_norm_rope(Y, norm_q, norm_k, rope, eps, head_dim):
    """Q/K head RMSNorm then pair rotation, V untouched, with plain loops.

    Y: list of rows of 3 C values; rope[m][i] = (cos, sin) for pair i.
    """
    out = [list(row) for row in Y]
    C = len(Y[0]) // 3
    for m, row in enumerate(Y):
        for part, w in ((0, norm_q), (1, norm_k)):
            for h0 in range(part * C, (part + 1) * C, head_dim):
                head = row[h0:h0 + head_dim]
                ms = math.fsum(v * v for v in head) / head_dim
                inv = 1.0 / math.sqrt(ms + eps)
                z = [head[d] * inv * w[d] for d in range(head_dim)]
                for i in range(head_dim // 2):
                    c, s = rope[m][i]
                    out[m][h0 + 2 * i] = z[2 * i] * c - z[2 * i + 1] * s
                    out[m][h0 + 2 * i + 1] = z[2 * i + 1] * c + z[2 * i] * s
    return out


def w4a16_forward(W, X, s, bias=None):
    """W4A16 layer on nested lists: W [N][K], X [M][K], s [K] (per input channel)."""
    N, K = len(W), len(W[0])
    Wp = [[f32r(W[n][j] * s[j]) for j in range(K)] for n in range(N)]
    g = global_scale(max(abs(v) for row in Wp for v in row))
    codes, scales = quantize_rows(Wp, g)
    dw = deq(codes, scales)
    inv = [f32r(1.0 / s[j]) for j in range(K)]
    Y = []
    for x in X:
        xt = [f16r(f32r(x[j] * inv[j])) for j in range(K)]
        row = []
        for n in range(N):
            y = g * math.fsum(xt[j] * dw[n][j] for j in range(K))
            if bias is not None:
                y += bias[n]
            row.append(y)
        Y.append(row)
    return dict(codes=codes, scales=scales, g=g, Y=Y)


# ---------------------------------------------------------------- INT4 variant


INT4 = [(Fraction(v), v) for v in range(-7, 8)]  # the symmetric 4-bit integer grid


def nearest_int4(x):
    """Nearest grid integer by exact rational distance, ties to the even integer."""
    a = Fraction(x)
    best = None
    for v, q in INT4:
        d = abs(a - v)
        if best is None or d < best[0] or (d == best[0] and q % 2 == 0):
            best = (d, q)
    return best[1]


def int4_quantize_rows(rows):
    """Per group of 64: s = bf16(f32(amax / 7)), q = nearest grid integer to f32(t * f32(1 / s))."""
    codes, scales = [], []
    for row in rows:
        rc, rs = [], []
        for b in range(0, len(row), 64):
            grp = row[b:b + 64]
            s = bf16r(f32r(max(abs(t) for t in grp) / 7.0))
            rcp = 0.0 if s == 0.0 else f32r(1.0 / s)
            rc += [nearest_int4(f32r(t * rcp)) for t in grp]
            rs.append(s)
        codes.append(rc)
        scales.append(rs)
    return codes, scales


def int4_layer_forward(W, X, act_amax, L1, L2, bias=None, gelu=False):
    """The INT4 layer on nested lists: smoothing and residual as layer_forward, INT4 quantizer,
    Y = sum over groups of s_a s_w (q_a . q_w) + (x_hat L1) L2 + b with exact rational sums."""
    N, K = len(W), len(W[0])
    M = len(X)
    r = len(L2)
    w_amax = [max(abs(W[n][j]) for n in range(N)) for j in range(K)]
    inv = []
    lam = []
    for j in range(K):
        a, w = act_amax[j], w_amax[j]
        lj = 1.0 if (a == 0.0 or w == 0.0) else f32r(math.sqrt(f32r(a / w)))
        lam.append(lj)
        inv.append(f32r(1.0 / lj))
    R = [[lam[j] * W[n][j] for n in range(N)] for j in range(K)]
    for i in range(r):
        for j in range(K):
            for n in range(N):
                R[j][n] = R[j][n] - L1[j][i] * L2[i][n]
    R32t = [[f32r(R[j][n]) for j in range(K)] for n in range(N)]
    wc, ws = int4_quantize_rows(R32t)
    xh = [[bf16r(f32r(X[m][j] * inv[j])) for j in range(K)] for m in range(M)]
    ac, as_ = int4_quantize_rows(xh)
    lr = [[sum(Fraction(xh[m][j]) * Fraction(L1[j][i]) for j in range(K)) for i in range(r)] for m in range(M)]
    Y = []
    for m in range(M):
        row = []
        for n in range(N):
            y = Fraction(0)
            for gi in range(K // 64):
                dot = sum(ac[m][k] * wc[n][k] for k in range(64 * gi, 64 * gi + 64))  # integers
                y += Fraction(as_[m][gi]) * Fraction(ws[n][gi]) * dot
            y += sum(lr[m][i] * Fraction(L2[i][n]) for i in range(r))
            if bias is not None:
                y += Fraction(bias[n])
            yf = float(y)
            if gelu:
                yf = 0.5 * yf * (1.0 + math.tanh(math.sqrt(2.0 / math.pi) * (yf + 0.044715 * yf ** 3)))
            row.append(yf)
        Y.append(row)
    return dict(lam=lam, inv=inv, w_codes=wc, w_scales=ws, a_codes=ac, a_scales=as_, x_hat=xh,
                lr=[[float(v) for v in row] for row in lr], Y=Y)
