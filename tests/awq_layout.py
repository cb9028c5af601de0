"""The awq_w4a16 GEMV's tile layout and its tensor-core data path, written out on the CPU from
their definitions (the library's pack kernel must produce the same bytes; the emulation checks
that the layout feeds m16n8k16 MMAs with the right operands)."""
import numpy as np


def tile_layout(q, s, z):
    """The GEMV's tile layout written out from its definition (rows padded to 16): word st of
    lane L = 4 g + t of tile (rb, G), nibble j = 4 h + i, holds
    q[16 rb + g + 8 (i & 1)][64 G + 16 st + 2 t + 8 (i >> 1) + h]; the tile's 64 side bytes hold,
    for each g, {s[row g], s[row g + 8], 128 + z[row g], 128 + z[row g + 8]} as fp16."""
    N, K = q.shape
    Np = (N + 15) // 16 * 16
    qp = np.zeros((Np, K), np.uint32)
    qp[:N] = q
    sp = np.zeros((Np, K // 64), np.float16)
    sp[:N] = s.astype(np.float16)
    zp = np.zeros((Np, K // 64), np.float16)  # 128 + z (rows past N: z = 0)
    zp[:] = 128
    zp[:N] = 128 + z.astype(np.float64)
    wt = np.zeros((Np // 16, K // 64, 32, 4), np.uint32)
    szt = np.zeros((Np // 16, K // 64, 8, 8), np.uint8)
    for L in range(32):
        g, t = L // 4, L % 4
        for st in range(4):
            for j in range(8):
                i, h = j % 4, j // 4
                rows = np.arange(Np // 16)[:, None] * 16 + g + 8 * (i & 1)
                ks = np.arange(K // 64)[None, :] * 64 + 16 * st + 2 * t + 8 * (i >> 1) + h
                wt[:, :, L, st] |= qp[rows, ks] << (4 * j)
    for g in range(8):
        r0 = np.arange(Np // 16) * 16 + g
        szt[:, :, g, 0:2] = sp[r0].view(np.uint8).reshape(Np // 16, K // 64, 2)
        szt[:, :, g, 2:4] = sp[r0 + 8].view(np.uint8).reshape(Np // 16, K // 64, 2)
        szt[:, :, g, 4:6] = zp[r0].view(np.uint8).reshape(Np // 16, K // 64, 2)
        szt[:, :, g, 6:8] = zp[r0 + 8].view(np.uint8).reshape(Np // 16, K // 64, 2)
    return wt.reshape(-1).view(np.uint8), szt.reshape(-1)




def xb_layout(X):
    """The GEMV's staged activations: word (G 32 + 4 m + t) 8 + 2 s + u holds the bf16 pair
    x[m][64 G + 16 s + 8 u + 2 t .. + 1] (8 token slots, zeros beyond M), as (lo, hi) values."""
    M, K = X.shape
    Xp = np.zeros((8, K))
    Xp[:M] = X
    out = np.zeros((K // 64, 32, 8, 2))
    for G in range(K // 64):
        for L in range(32):
            m, t = L // 4, L % 4
            for v in range(8):
                st, u = v // 2, v % 2
                k = 64 * G + 16 * st + 8 * u + 2 * t
                out[G, L, v] = Xp[m, k:k + 2]
    return out


def emulate_gemv(X, q, s, z):
    """The GEMV as the kernel computes it, in fp64: per tile, lane (g, t) turns word st of its 16
    bytes into A registers i = 0..3 with halves (128 + nibble i, 128 + nibble i + 4); the MMA's
    fragments place register i at rows g + 8 (i & 1), columns 2 t + 8 (i >> 1) + (0, 1), and B
    registers b0 / b1 at columns (rows of B) 2 t + (0, 1) / 2 t + 8 + (0, 1), token g; then
    acc += s (D - (128 + z) sum_G(x)). Returns Y (M x N) without bias."""
    M, K = X.shape
    N = q.shape[0]
    wt, szt = tile_layout(q, s, z)
    RB, GP = (N + 15) // 16, K // 64
    words = wt.view(np.uint32).reshape(RB, GP, 32, 4)
    side = szt.reshape(RB, GP, 8, 8)
    xb = xb_layout(X)
    Y = np.zeros((8, RB * 16))
    for rb in range(RB):
        acc = np.zeros((16, 8))
        for G in range(GP):
            D = np.zeros((16, 8))
            for st in range(4):
                A = np.zeros((16, 16))
                B = np.zeros((16, 8))
                for L in range(32):
                    g, t = L // 4, L % 4
                    w = int(words[rb, G, L, st])
                    for i in range(4):
                        lo, hi = 128 + ((w >> (4 * i)) & 0xF), 128 + ((w >> (4 * i + 16)) & 0xF)
                        r, c = g + 8 * (i & 1), 2 * t + 8 * (i >> 1)
                        A[r, c], A[r, c + 1] = lo, hi
                    b = xb[G, L]
                    B[2 * t:2 * t + 2, g] = b[2 * st]
                    B[2 * t + 8:2 * t + 10, g] = b[2 * st + 1]
                D += A @ B
            for g in range(8):
                sv = side[rb, G, g].view(np.float16).astype(np.float64)
                sx = np.array([xb[G, 4 * m:4 * m + 4].sum() for m in range(8)])
                for h in range(2):
                    r = g + 8 * h
                    acc[r] += sv[h] * (D[r] - sv[2 + h] * sx)
        Y[:, 16 * rb:16 * rb + 16] = acc.T
    return Y[:M, :N]
