"""Search the token order inside a 16-token decode subtile that minimises
shared-memory wavefronts of the decode kernel's code loads.

In decode_kernel a warp reads the packed rows of a 16-token subtile from the
staged chunk: for the scores, lane (g, t) reads the K rows of MMA rows g and
g + 8 (its quarter t of the coordinates); for the V accumulation it reads the
V rows of MMA columns 2t, 2t+1, 2t+8, 2t+9 (its eighth g of the coordinates).
Rows are 24..64 bytes, so these loads hit the same banks from several rows.
MMA row/column k may hold any physical token pi[k] of the subtile, as long as
K and V use the same order; this script models the loads (the same shapes as
KChunk::load / VChunk::load, 32 banks of 4 bytes, 64-bit loads served in two
half-warp passes and 128-bit loads in four) and anneals pi per format pair.
It prints the kTokenPerm table used by tq_attn.cu.  Run: python bank_perm.py
"""
import math
import random


def fmt(mse, mixed=False, prod=False):
    return dict(mse=mse, mixed=mixed, prod=prod,
                code=8 * (2 * mse + 1) if mixed else 16 * mse,
                segs=([(mse + 1, 64, 0), (mse, 64, 8 * (mse + 1))] if mixed else ([(mse, 128, 0)] if mse else [])))


def wavefronts(addrs, width):
    per = 32 // (width // 4)
    total = 0
    for p in range(0, 32, per):
        banks = {}
        for lane in range(p, p + per):
            a = addrs[lane]
            if a is None:
                continue
            for w in range(width // 4):
                word = a // 4 + w
                banks.setdefault(word % 32, set()).add(word)
        if banks:
            total += max(len(s) for s in banks.values())
    return total


LANES = [(lane >> 2, lane & 3) for lane in range(32)]


def k_loads(f, rows, plane_base):
    """(address list, width) of the K loads of one row set (one per lane)."""
    out = []
    for b, nd, byte0 in f["segs"]:
        nbytes = nd * b // 32
        for g_t_off in range(1):
            o = [byte0 + t * nbytes for g, t in LANES]
            base = [plane_base + rows[g] * f["code"] for g, t in LANES]
            if nbytes == 16:
                out.append(([x + y for x, y in zip(base, o)], 16))
            elif nbytes == 12:
                for d in (0, 4, 8):
                    out.append(([x + y + d for x, y in zip(base, o)], 4))
            elif nbytes == 8:
                out.append(([x + y for x, y in zip(base, o)], 8))
            elif nbytes == 6:
                for d in (0, 4):
                    out.append(([x + (y & ~3) + d for x, y in zip(base, o)], 4))
            elif nbytes == 4:
                out.append(([x + y for x, y in zip(base, o)], 4))
            else:
                raise ValueError(nbytes)
    return out


def v_loads(f, rows_of_t, plane_base):
    out = []
    for b, nd, byte0 in f["segs"]:
        bits = nd * b // 8
        base = [plane_base + rows_of_t[t] * f["code"] for g, t in LANES]
        if bits == 64:
            out.append(([x + byte0 + 8 * g for x, (g, t) in zip(base, LANES)], 8))
        elif bits == 32:
            out.append(([x + byte0 + 4 * g for x, (g, t) in zip(base, LANES)], 4))
        elif bits == 16:
            out.append(([x + ((byte0 + 2 * g) & ~3) for x, (g, t) in zip(base, LANES)], 4))
        elif bits == 48:
            for d in (0, 4):
                out.append(([x + ((byte0 + 6 * g) & ~3) + d for x, (g, t) in zip(base, LANES)], 4))
        elif bits == 24:
            o = [byte0 + 3 * g for g, t in LANES]
            out.append(([x + (y & ~3) for x, y in zip(base, o)], 4))
            out.append(([x + (y & ~3) + 4 if (y & 3) * 8 > 8 else None for x, y in zip(base, o)], 4))
        else:
            raise ValueError(bits)
    return out


def stage_bases(fk, fv, chunk):
    kc = 0
    vc = kc + chunk * fk["code"]
    kn = vc + chunk * fv["code"]
    vn = kn + chunk * 4
    kq = vn + chunk * 4
    kr = kq + (chunk * 16 if fk["prod"] else 0)
    vq = kr + (chunk * 4 if fk["prod"] else 0)
    return kc % 128, vc % 128, kq % 128, vq % 128


def cost(pi, fk, fv, chunk):
    kc, vc, kq, vq = stage_bases(fk, fv, chunk)
    total = 0
    for half in (0, 8):
        rows = [pi[g + half] for g in range(8)]
        for addrs, w in k_loads(fk, rows, kc):
            total += wavefronts(addrs, w)
        if fk["prod"]:
            total += wavefronts([kq + rows[g] * 16 + 4 * t for g, t in LANES], 4)
    for c in (0, 1, 8, 9):
        rows_of_t = [pi[2 * t + c] for t in range(4)]
        for addrs, w in v_loads(fv, rows_of_t, vc):
            total += wavefronts(addrs, w)
        if fv["prod"]:
            total += wavefronts([vq + rows_of_t[t] * 16 + ((2 * g) & ~3) for g, t in LANES], 4)
    return total


def search(fk, fv, chunk, seed=1, restarts=8, iters=20000):
    rng = random.Random(seed)
    best = list(range(16))
    bc = cost(best, fk, fv, chunk)
    for _ in range(restarts):
        p = list(range(16))
        rng.shuffle(p)
        c = cost(p, fk, fv, chunk)
        temp = 3.0
        for _ in range(iters):
            q = p[:]
            i, j = rng.sample(range(16), 2)
            q[i], q[j] = q[j], q[i]
            cq = cost(q, fk, fv, chunk)
            if cq <= c or rng.random() < math.exp((c - cq) / temp):
                p, c = q, cq
            temp = max(0.05, temp * 0.9997)
            if c < bc:
                best, bc = p[:], c
    return best, bc


# (K format id, V format id, format dicts, tokens per chunk) of the kernel
# instantiations; ids as in tq_attn.cu: mse | mixed << 3 | prod << 4
PAIRS = [
    (1, 1, fmt(1), fmt(1), 480), (2, 2, fmt(2), fmt(2), 480), (3, 3, fmt(3), fmt(3), 480),
    (4, 4, fmt(4), fmt(4), 240), (11, 11, fmt(3, True), fmt(3, True), 480), (10, 10, fmt(2, True), fmt(2, True), 480),
    (16, 16, fmt(0, prod=True), fmt(0, prod=True), 480), (17, 17, fmt(1, prod=True), fmt(1, prod=True), 480),
    (18, 18, fmt(2, prod=True), fmt(2, prod=True), 480), (19, 19, fmt(3, prod=True), fmt(3, prod=True), 480),
    (4, 3, fmt(4), fmt(3), 480), (4, 2, fmt(4), fmt(2), 240), (3, 2, fmt(3), fmt(2), 480),
]

if __name__ == "__main__":
    for kf, vf, fk, fv, chunk in PAIRS:
        ident = cost(list(range(16)), fk, fv, chunk)
        best, bc = search(fk, fv, chunk)
        word = sum(v << (4 * k) for k, v in enumerate(best))
        print(f"  {{{kf}, {vf}, 0x{word:016X}ull}},  // wavefronts per subtile {ident} -> {bc}")
