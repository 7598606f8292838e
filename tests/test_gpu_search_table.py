"""The search tables built on the GPU list, for every cell, a superset of the
codewords that can win there: for many directions x (random, on cell
boundaries, on Voronoi boundaries between codewords) the exact fp64 argmax of
<x, c> over all 24 S codewords is in the list of x's cell, computed here
independently in numpy from the table's documented layout (face = first
coordinate a of largest |x_a| and the sign of x_a; gnomonic coordinates t =
the other three coordinates in index order / |x_a|; u = t (A + B t^2) with
A = fp32(4/pi), B = 1 - A; 8 faces x 32^3 cells in u; 8 uint16 slots holding
12-bit candidate ids in increasing order, the top 4 bits of slot 0 holding the
count, 0 = overflow).  A point within 1e-6 of a cell face is checked against
the cells on both sides (the kernel's fp32 arithmetic may pick either)."""
import itertools
import numpy as np
import pytest
import torch

from _parity import gpu_search_table, to_host

pytestmark = pytest.mark.gpu
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

G = 32
A = float(np.float32(4.0 / np.pi))
B = float(np.float32(1.0 - np.float32(A)))


def face_coords(x):
    """(face 2 a + (x_a < 0), t = the other coordinates in order / |x_a|)."""
    a = np.argmax(np.abs(x), axis=1)
    rows = np.arange(len(x))
    xa = x[rows, a]
    others = np.array([[k for k in range(4) if k != ax] for ax in range(4)])[a]
    t = np.take_along_axis(x, others, axis=1) / np.abs(xa)[:, None]
    return 2 * a + (xa < 0), t


def u_of_t(t):
    return t * (A + B * t * t)


def t_of_u(u):
    lo, hi = -np.ones_like(u), np.ones_like(u)
    for _ in range(60):
        m = 0.5 * (lo + hi)
        below = u_of_t(m) < u
        lo, hi = np.where(below, m, lo), np.where(below, hi, m)
    return 0.5 * (lo + hi)


def cell_candidates(face, t, eps=1e-6):
    """All table entries the point may land in: per axis floor of (u +- eps)."""
    u = u_of_t(t)
    lo = np.clip(np.floor((u - eps + 1.0) * (G / 2)).astype(int), 0, G - 1)
    hi = np.clip(np.floor((u + eps + 1.0) * (G / 2)).astype(int), 0, G - 1)
    out = []
    for pick in itertools.product((0, 1), repeat=3):
        i = np.where(np.array(pick) == 1, hi, lo)
        out.append(face * G ** 3 + (i[:, 0] * G + i[:, 1]) * G + i[:, 2])
    return out


@pytest.mark.parametrize("S", [8, 32, 48])
def test_table_lists_contain_the_exact_argmax(oracle, S):
    cb = oracle.make_codebook(5, S, 1)
    tab = to_host(gpu_search_table(torch.from_numpy(cb.reshape(-1)).cuda(), S, 1))
    raw = tab.view(np.uint16).reshape(8 * G ** 3, 8).astype(np.int64)
    count = raw[:, 0] >> 12
    overflow = count == 0
    rec = raw & 0xFFF
    rec[np.arange(8)[None, :] >= count[:, None]] = 0xFFFF    # past the count: not listed
    assert np.all(count <= 8) and np.all(rec[:, 0] < 24 * S)
    # listed ids increase (equal scores then keep the lowest index); padding = 24 S
    listed = np.where(rec == 0xFFFF, 1 << 20, rec)[~overflow]
    assert np.all((np.diff(listed, axis=1) > 0) | (listed[:, 1:] == 1 << 20))
    pad = (raw & 0xFFF)[~overflow][rec[~overflow] == 0xFFFF]
    assert np.all(pad == 24 * S)
    assert overflow.mean() < 0.01
    cw = np.array([oracle.codeword(i % 24, cb[0, i // 24]) for i in range(24 * S)], np.float64)
    rng = np.random.default_rng(S)
    xs = [rng.standard_normal((200000, 4))]
    # points whose coordinates sit on cell boundaries, on every face
    b = rng.integers(0, G + 1, (20000, 3))
    t = t_of_u(-1.0 + 2.0 * b / G)
    xb = np.concatenate([np.ones((20000, 1)), t], 1) * rng.choice([-1, 1], (20000, 1))
    xs.append(np.take_along_axis(xb, np.argsort(rng.random((20000, 4)), axis=1), axis=1))
    # points on the bisector of two neighbouring codewords (exact ties)
    i, j = rng.integers(0, 24 * S, (2, 20000))
    xs.append(cw[i] + cw[j])
    x = np.concatenate(xs).astype(np.float32).astype(np.float64)
    x = x[np.linalg.norm(x, axis=1) > 1e-3]
    face, t = face_coords(x)
    sc = x @ cw.T
    best = sc.max(1, keepdims=True)
    winners = sc >= best - 1e-12 * np.abs(best)       # every (near-)exact argmax
    n_checked = 0
    rows = np.arange(len(x))
    for cell in cell_candidates(face, t):
        lists = rec[cell]
        ok = overflow[cell].copy()
        for k in range(8):
            lk = lists[:, k]
            ok |= (lk < 24 * S) & winners[rows, np.minimum(lk, 24 * S - 1)]
        assert ok.all(), "argmax missing from %d cell lists" % (~ok).sum()
        n_checked += len(cell)
    print("[table] S=%d: %d lookups, overflow cells %.3f%%, mean list %.2f"
          % (S, n_checked, 100 * overflow.mean(),
             (rec[~overflow] != 0xFFFF).sum(1).mean()))
