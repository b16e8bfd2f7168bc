"""The NVFP4 storage layout declared in include/beam_moe.h, written out element by element, read
back by the test helpers that unpack the CUDA path's weights (no GPU needed)."""
import numpy as np

from tests import gpu_helpers as H


def _pack(codes, bs, interleave_rows=None):
    """Packs codes [rows, cols] and block scales [rows, cols / 16] the way the header states:
    two codes per byte (element 2i in the low nibble), scales at byte
    ((g * cols / 64 + j / 4) * 512) + (r % 32) * 16 + (r / 32) * 4 + j % 4 for row 128g + r."""
    rows, cols = codes.shape
    packed = np.zeros((rows, cols // 2), np.uint8)
    for i in range(cols // 2):
        packed[:, i] = codes[:, 2 * i] | (codes[:, 2 * i + 1] << 4)
    atoms = np.zeros(rows * cols // 16, np.uint8)
    for row in range(rows):
        g, r = divmod(row, 128)
        for j in range(cols // 16):
            atoms[(g * cols // 64 + j // 4) * 512 + (r % 32) * 16 + (r // 32) * 4 + j % 4] = bs[row, j]
    return packed, atoms


def test_unpack_and_atoms_read_back_the_documented_layout():
    rng = np.random.default_rng(0)
    rows, cols = 256, 512
    codes = rng.integers(0, 16, (rows, cols)).astype(np.uint8)
    bs = rng.integers(0, 256, (rows, cols // 16)).astype(np.uint8)
    packed, atoms = _pack(codes, bs)
    assert np.array_equal(H.unpack_e2m1(packed), codes)
    assert np.array_equal(H.atoms_to_rows(atoms, rows, cols), bs)


def test_interleaved_gate_up_rows_split_back():
    """Output row 128c + w of the interleaved gate|up matrix is gate row 64c + w (w < 64) or up
    row 64c + w - 64."""
    import torch
    rng = np.random.default_rng(1)
    E, I, d = 2, 128, 256
    gate = rng.integers(0, 16, (E, I, d)).astype(np.uint8)
    up = rng.integers(0, 16, (E, I, d)).astype(np.uint8)
    gbs = rng.integers(0, 256, (E, I, d // 16)).astype(np.uint8)
    ubs = rng.integers(0, 256, (E, I, d // 16)).astype(np.uint8)
    gs = rng.random((E, I)).astype(np.float32)
    us = rng.random((E, I)).astype(np.float32)
    down = rng.integers(0, 16, (E, d, I)).astype(np.uint8)
    dbs = rng.integers(0, 256, (E, d, I // 16)).astype(np.uint8)
    ds = rng.random((E, d)).astype(np.float32)
    gu_c, gu_a, gu_s, dn_c, dn_a = [], [], [], [], []
    for e in range(E):
        rows_c = np.empty((2 * I, d), np.uint8)
        rows_b = np.empty((2 * I, d // 16), np.uint8)
        rows_s = np.empty(2 * I, np.float32)
        for p in range(2 * I):
            c, w = divmod(p, 128)
            src, sb, ss = (gate, gbs, gs) if w < 64 else (up, ubs, us)
            rows_c[p], rows_b[p], rows_s[p] = src[e, 64 * c + w % 64], sb[e, 64 * c + w % 64], ss[e, 64 * c + w % 64]
        pc, pa = _pack(rows_c, rows_b)
        gu_c.append(pc), gu_a.append(pa), gu_s.append(rows_s)
        qc, qa = _pack(down[e], dbs[e])
        dn_c.append(qc), dn_a.append(qa)
    w4 = ((torch.from_numpy(np.stack(gu_c)), torch.from_numpy(np.stack(gu_a)),
           torch.from_numpy(np.stack(gu_s))),
          (torch.from_numpy(np.stack(dn_c)), torch.from_numpy(np.stack(dn_a)), torch.from_numpy(ds)))
    for e in range(E):
        (qg, bg, sg), (qu, bu, su), (qd, bd, sd) = H.nvfp4_expert_from_device(w4, e, I, d)
        assert np.array_equal(qg, gate[e]) and np.array_equal(qu, up[e])
        assert np.array_equal(bg, gbs[e]) and np.array_equal(bu, ubs[e])
        assert np.array_equal(sg, gs[e]) and np.array_equal(su, us[e])
        assert np.array_equal(qd, down[e]) and np.array_equal(bd, dbs[e]) and np.array_equal(sd, ds[e])
