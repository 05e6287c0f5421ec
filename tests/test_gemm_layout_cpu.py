"""Host-side replay of the tcgen05 grouped GEMM's shared-memory layout and
epilogue store arithmetic (recurrent_memory_transformer_diag_b200/csrc/tc_gemm.cu),
with the layout constants read from the kernel source:

* every CTA's shared memory (pipeline stages, barriers, the transposed ragged
  tile's staging area, the per-warp 16-bit output slots) fits the 227 KB a
  CTA may have, with the worst-case slack of aligning the base to 1024 bytes;
* the reader lanes of a transposed ragged tile stay inside the staging area
  (lanes past the staged rows read row 0);
* the slot stores of the QKV, residual and SwiGLU epilogues write only rows
  < M and columns < the output width, for the configurations the forward runs.
"""
import itertools
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "recurrent_memory_transformer_diag_b200", "csrc", "tc_gemm.cu")
CTA_SMEM = 227 * 1024


def _const(text, name):
    m = re.search(r"constexpr int %s = (\d+);" % name, text)
    assert m, name
    return int(m.group(1))


@pytest.fixture(scope="module")
def k():
    text = open(SRC).read()
    c = {n: _const(text, n) for n in ("BM", "BK", "EPI_WARPS", "SWAP_ROWS", "XS_SLOT")}
    m = re.search(r"STAGES = BN >= 256 \? (\d+) : \(BN >= 128 \? (\d+) : (\d+)\)", text)
    assert m, "stage rule"
    c["stages"] = tuple(int(x) for x in m.groups())
    # the reader clamp of the transposed tile
    assert "lane < SWAP_ROWS ? lane : 0" in text
    return c


def layout(k, BN):
    st256, st128, st64 = k["stages"]
    stages = st256 if BN >= 256 else (st128 if BN >= 128 else st64)
    stage_bytes = k["BM"] * k["BK"] * 2 + BN * k["BK"] * 2
    bar = stages * stage_bytes
    swap = BN % 128 == 0
    stg_off = bar + 256
    pitch = BN + 4
    stg_bytes = k["SWAP_ROWS"] * pitch * 4 if swap else 0
    xs_off = stg_off + stg_bytes
    total = xs_off + k["EPI_WARPS"] * k["XS_SLOT"] + 1024
    return dict(stg_off=stg_off, pitch=pitch, stg_bytes=stg_bytes, xs_off=xs_off, total=total, swap=swap)


@pytest.mark.parametrize("BN", [64, 128, 256])
def test_shared_memory_fits_and_accesses_stay_inside(k, BN):
    L = layout(k, BN)
    static = 16
    assert L["total"] + static <= CTA_SMEM
    usable = L["total"] - 1008          # after aligning a 16-byte-aligned base up to 1024
    # per-warp output slots
    assert L["xs_off"] % 16 == 0 and L["xs_off"] + k["EPI_WARPS"] * k["XS_SLOT"] <= usable
    if L["swap"]:
        for lane in range(32):
            row = lane if lane < k["SWAP_ROWS"] else 0
            last = L["stg_off"] + (row * L["pitch"] + BN - 1) * 4 + 3
            assert last < L["stg_off"] + L["stg_bytes"], lane
        assert (L["pitch"] * 4) % 16 == 0          # 16-byte row reads


def _stores(k, M, N, out_cols, BN, epi, hd=64):
    """(row, col) pieces the slot stores write for one node of M rows."""
    BM = k["BM"]
    m_tiles = (M + BM - 1) // BM
    n_tiles = (N + BN - 1) // BN
    swap_tail = BN % 128 == 0 and M - (m_tiles - 1) * BM <= k["SWAP_ROWS"]
    for nb, mb in itertools.product(range(n_tiles), range(m_tiles)):
        swapped = swap_tail and mb == m_tiles - 1
        for warp in range(2, 2 + k["EPI_WARPS"]):
            quarter, half = warp & 3, (warp - 2) >> 2
            if swapped and quarter != 0:
                continue
            wrow0 = mb * BM + quarter * 32
            nrows = min(32, M - wrow0)
            if epi == "swiglu":
                chunks = [nb * (BN // 2) + c * 32 for c in range(half * (BN // 128), (half + 1) * (BN // 128))]
            elif epi == "qkv":
                hh_n, cph, pairs = BN // hd // 2, hd // 32, hd // 64
                chunks = [nb * BN + (hh * cph + pc + e * pairs) * 32
                          for hh in range(half * hh_n, (half + 1) * hh_n) for pc in range(pairs) for e in (0, 1)]
            else:
                chunks = [nb * BN + (half * (BN // 64) + q) * 32 for q in range(BN // 64)]
            for col in chunks:
                if col >= out_cols:
                    continue
                nv = out_cols - col
                for r in range(32):
                    for q in range(4):
                        if r < nrows and 8 * q < nv:
                            yield wrow0 + r, col + 8 * q


@pytest.mark.parametrize("name,Tp,d,F,nqkv,hd", [
    ("small", 144, 256, 688, 768, 64), ("small short", 40, 256, 688, 768, 64),
    ("1b", 1040, 2048, 8192, 3072, 64), ("3b", 2064, 3072, 8192, 5120, 128)])
def test_slot_stores_stay_in_rows_and_columns(k, name, Tp, d, F, nqkv, hd):
    f_pad = (F + 127) // 128 * 128
    for N, out_cols, epi in ((nqkv, nqkv, "qkv"), (d, d, "resid"), (2 * f_pad, F, "swiglu")):
        for r, c in _stores(k, Tp, N, out_cols, 256, epi, hd):
            assert 0 <= r < Tp and c + 8 <= out_cols, (name, epi, r, c)
