"""Host model of the append kernel's store phase (csrc/kvq_kernels.cu).

A window of 16 input tokens is staged in shared memory and written out in one
of two ways; this file restates both on the host and checks them against the
plain per-token layout of the cache pages:

* A window that fills one page in order leaves V transposed through byte
  permutes: two 4x4 byte transposes per 8-byte piece (8-bit codes) or 2x2
  transposes of 16-bit halves (BF16). The model of the permute follows its
  definition (each result byte picks one of the 8 bytes of the two operands by
  a selector nibble).
* Any other window is cut into segments (runs of consecutive slots inside one
  page); each (segment, channel, 16-byte chunk) writes its byte range once, as
  aligned 16/8/4/2/1-byte pieces that cover exactly that range.

V page layout: (token t, channel d) at byte (t*E // 16) * D * 16 + d * 16 +
(t*E) % 16, E the element size.
"""

import numpy as np

BS = 16


def byte_perm(x, y, sel):
    b = [(x >> (8 * i)) & 0xFF for i in range(4)] + [(y >> (8 * i)) & 0xFF for i in range(4)]
    return sum(b[(sel >> (4 * i)) & 7] << (8 * i) for i in range(4))


def word(buf, off):
    return int.from_bytes(bytes(buf[off:off + 4]), "little")


def v_offset(t, d, D, E):
    return (t * E // 16) * D * 16 + d * 16 + (t * E) % 16


def pieces16(p, e):
    """(offset, size) stores the kernel issues for bytes [p, e) of a chunk."""
    if p == 0 and e == 16:
        return [(0, 16)]
    out = []
    for h8 in range(2):
        a8, b8 = max(p, 8 * h8), min(e, 8 * h8 + 8)
        if a8 >= b8:
            continue
        if a8 == 8 * h8 and b8 == 8 * h8 + 8:
            out.append((8 * h8, 8))
            continue
        for h4 in range(2):
            base4 = 8 * h8 + 4 * h4
            a4, b4 = max(a8, base4), min(b8, base4 + 4)
            if a4 >= b4:
                continue
            if a4 == base4 and b4 == base4 + 4:
                out.append((base4, 4))
                continue
            for h2 in range(2):
                base2 = base4 + 2 * h2
                a2, b2 = max(a4, base2), min(b4, base2 + 2)
                if a2 >= b2:
                    continue
                out.append((base2, 2) if (a2 == base2 and b2 == base2 + 2) else (a2, 1))
    return out


def test_piece_decomposition_covers_exactly_with_aligned_stores():
    for p in range(16):
        for e in range(p + 1, 17):
            ps = pieces16(p, e)
            covered = sorted(b for o, n in ps for b in range(o, o + n))
            assert covered == list(range(p, e))
            assert all(o % n == 0 for o, n in ps)


def test_whole_page_transposes():
    rng = np.random.default_rng(1)
    for D in (64, 128):
        for E in (1, 2):
            pad = D * E + 16
            vbuf = rng.integers(0, 256, 16 * pad, dtype=np.uint8)
            page = np.zeros(16 * D * E, np.uint8)
            if E == 1:
                for j in range(2 * (D // 4)):
                    c, hh = j % (D // 4), j // (D // 4)
                    o = [[0, 0] for _ in range(4)]
                    for g in range(2):
                        t0 = 8 * hh + 4 * g
                        r = [word(vbuf, (t0 + i) * pad + 4 * c) for i in range(4)]
                        a01, a23 = byte_perm(r[0], r[1], 0x5140), byte_perm(r[2], r[3], 0x5140)
                        b01, b23 = byte_perm(r[0], r[1], 0x7362), byte_perm(r[2], r[3], 0x7362)
                        o[0][g], o[1][g] = byte_perm(a01, a23, 0x5410), byte_perm(a01, a23, 0x7632)
                        o[2][g], o[3][g] = byte_perm(b01, b23, 0x5410), byte_perm(b01, b23, 0x7632)
                    for m in range(4):
                        off = (4 * c + m) * 16 + 8 * hh
                        page[off:off + 8] = np.frombuffer(
                            o[m][0].to_bytes(4, "little") + o[m][1].to_bytes(4, "little"), np.uint8)
            else:
                for j in range(2 * (D // 2)):
                    c, u = j % (D // 2), j // (D // 2)
                    lo, hi = [], []
                    for q in range(4):
                        t0 = 8 * u + 2 * q
                        w0, w1 = word(vbuf, t0 * pad + 4 * c), word(vbuf, (t0 + 1) * pad + 4 * c)
                        lo.append(byte_perm(w0, w1, 0x5410))
                        hi.append(byte_perm(w0, w1, 0x7632))
                    for ch, ws in ((2 * c, lo), (2 * c + 1, hi)):
                        off = (u * D + ch) * 16
                        page[off:off + 16] = np.frombuffer(b"".join(x.to_bytes(4, "little") for x in ws), np.uint8)
            want = np.zeros_like(page)
            for t in range(16):
                for d in range(D):
                    o = v_offset(t, d, D, E)
                    want[o:o + E] = vbuf[t * pad + d * E:t * pad + d * E + E]
            assert np.array_equal(page, want), (D, E)


def _segments(sl, nslots):
    valid = [0 <= s < nslots for s in sl]
    start = [valid[i] and not (i > 0 and valid[i - 1] and sl[i] == sl[i - 1] + 1 and sl[i] % BS != 0)
             for i in range(16)]
    segs = []
    for i in range(16):
        if start[i]:
            j = i + 1
            while j < 16 and valid[j] and not start[j]:
                j += 1
            segs.append((i, j - i))
    return segs


def test_segment_stores_equal_per_token_stores():
    rng = np.random.default_rng(0)
    for trial in range(1500):
        D = int(rng.choice([64, 128]))
        E = int(rng.choice([1, 2]))
        NB = int(rng.integers(2, 6))
        n = int(rng.integers(1, 17))
        kind = trial % 4
        if kind == 0:
            s0 = int(rng.integers(0, NB * BS - n + 1))
            slots = list(range(s0, s0 + n))
        elif kind == 1:
            slots = [int(x) for x in rng.permutation(NB * BS)[:n]]
        elif kind == 2:
            s0 = int(rng.integers(0, NB * BS - n + 1))
            slots = list(range(s0, s0 + n))
            for _ in range(3):
                slots[int(rng.integers(0, n))] = int(rng.choice([-1, NB * BS + 3]))
        else:
            a, b = int(rng.integers(0, NB * BS - 16)), int(rng.integers(0, NB * BS - 16))
            m = int(rng.integers(0, n + 1))
            slots = list(range(a, a + m)) + list(range(b, b + n - m))
        ok = [s for s in slots if 0 <= s < NB * BS]
        if len(set(ok)) < len(ok):
            continue                                   # slots must be distinct within a call
        sl = slots + [-1] * (16 - n)
        pad = D * E + 16
        vbuf = rng.integers(0, 256, (16, pad), dtype=np.uint8)
        pageb = BS * D * E
        got = np.full(NB * pageb, 0xAA, np.uint8)
        want = got.copy()
        tpc = 16 // E
        for i0, ln in _segments(sl, NB * BS):
            o0 = sl[i0] % BS
            base = (sl[i0] // BS) * pageb
            for d in range(D):
                for u in range(E):
                    ta, tz = max(o0, u * tpc), min(o0 + ln, (u + 1) * tpc)
                    if ta >= tz:
                        continue
                    chunk = base + (u * D + d) * 16
                    for off, size in pieces16((ta - u * tpc) * E, (tz - u * tpc) * E):
                        for byte in range(off, off + size):
                            t = u * tpc + byte // E
                            i = i0 + (t - o0)
                            got[chunk + byte] = vbuf[i, d * E + byte % E]
        for i, s in enumerate(sl):
            if 0 <= s < NB * BS:
                base = (s // BS) * pageb
                for d in range(D):
                    o = base + v_offset(s % BS, d, D, E)
                    want[o:o + E] = vbuf[i, d * E:d * E + E]
        assert np.array_equal(got, want)
