"""Index arithmetic of the multi-token kernel (csrc/gdn_decode_mt.cu), restated on the
host for every supported shape, so that a change which would send a copy out of its
buffer, misalign it, or leave a state element uncovered fails here, before any GPU run.
The formulas below are the kernel's own (shared-memory layout, staged copies, register
tile, history write); keep them in step with it."""
import itertools

import pytest

R16 = lambda x: (x + 15) // 16 * 16  # noqa: E731
SMEM_LIMIT = 232448                  # dynamic shared memory one CTA may use (227 KB)
CHUNK = 16384                        # bytes per state-tile bulk copy


def geometry(dk, dv):
    nwh = dv // 16
    nhc = min(16 // nwh, 8)
    return dict(NWH=nwh, NHC=nhc, NW=nwh * nhc, RPL=dk // 8, NCHC=2 * dk + nhc * dv, TILE=dk * dv * 4)


def layout(dk, dv, W, T):
    g = geometry(dk, dv)
    rows = g["NHC"] * g["TILE"]
    wts = rows + R16((W - 1 + T) * g["NCHC"] * 2)
    qk = wts + R16(g["NCHC"] * W * 2)
    vs = qk + T * 2 * dk * 4
    zb = vs + T * g["NHC"] * dv * 4
    sc = zb + T * g["NHC"] * dv * 2
    ctl = R16(sc + T * g["NHC"] * 20)
    return dict(rows=rows, wts=wts, qk=qk, vs=vs, zb=zb, sc=sc, ctl=ctl, total=ctl + 48)


def heads_per_pass(G, nhc):
    return max(d for d in range(1, min(G, nhc) + 1) if G % d == 0)


SHAPES = list(itertools.product((16, 32, 64, 128), (16, 32, 64, 128), (2, 3, 4, 8), (1, 5, 16), (1, 2, 3, 8)))


@pytest.mark.parametrize("dk,dv,W,T,G", SHAPES)
def test_multitoken_kernel_copies_stay_in_bounds(dk, dv, W, T, G):
    Hk = 2
    Hv = Hk * G
    C = 2 * Hk * dk + Hv * dv
    g, L = geometry(dk, dv), layout(dk, dv, W, T)
    assert L["total"] <= SMEM_LIMIT
    for k in ("rows", "wts", "qk", "vs", "zb"):
        assert L[k] % 16 == 0
    assert (L["ctl"] + 8) % 8 == 0
    NH = heads_per_pass(G, g["NHC"])
    npass, NCH = G // NH, 2 * dk + NH * dv
    for hk, ps, ntok in itertools.product(range(Hk), range(npass), {0, 1, T}):
        h0 = hk * G + ps * NH
        ch = (hk * dk, Hk * dk + hk * dk, 2 * Hk * dk + h0 * dv)
        # state tiles: warp w issues chunks w, w + NW, ... of the NH contiguous tiles
        tile_bytes = NH * g["TILE"]
        chunks = sorted(c for w in range(g["NW"]) for c in range(w * CHUNK, tile_bytes, g["NW"] * CHUNK))
        assert chunks == list(range(0, tile_bytes, CHUNK)) and tile_bytes <= L["rows"]
        assert all((h0 * dk * dv * 4 + c) % 16 == 0 and min(CHUNK, tile_bytes - c) % 16 == 0 for c in chunks)
        # staged raw rows (history, then the tokens) and weights: 16-byte asynchronous copies
        nv, nrow = NCH // 8, W - 1 + ntok
        for i in range(nrow * nv):
            r, lc = divmod(i, nv)
            lc *= 8
            run = 0 if lc < dk else (1 if lc < 2 * dk else 2)
            assert run == (0 if lc + 7 < dk else (1 if lc + 7 < 2 * dk else 2))  # never straddles two runs
            c0 = ch[run] + lc - (0, dk, 2 * dk)[run]
            assert c0 % 8 == 0 and c0 + 8 <= C
            assert (r * NCH + lc + 8) * 2 <= L["wts"] - L["rows"]
        for i in range(NCH * W // 8):
            lc, last = (i * 8) // W, (i * 8 + 7) // W
            run = 0 if lc < dk else (1 if lc < 2 * dk else 2)
            assert run == (0 if last < dk else (1 if last < 2 * dk else 2))
            c0 = ch[run] + lc - (0, dk, 2 * dk)[run]
            assert (c0 * W + (i * 8 - lc * W)) % 8 == 0 and (c0 + (last - lc) + 1) * W <= C * W
            assert (i * 8 + 8) * 2 <= L["qk"] - L["wts"]
        # z rows of the pass and the history write
        assert ntok * NH * dv * 2 <= L["sc"] - L["zb"] and (NH * dv * 2) % 16 == 0
        lc0 = 0 if ps == npass - 1 else 2 * dk
        for i in range((W - 1) * ((NCH - lc0) // 8)):
            r, lc = divmod(i, (NCH - lc0) // 8)
            lc = lc0 + lc * 8
            assert ntok + r < nrow and lc + 8 <= NCH  # a staged row: the last W-1 of history + tokens


@pytest.mark.parametrize("dk,dv", list(itertools.product((16, 32, 64, 128), (16, 32, 64, 128))))
def test_multitoken_register_tile_covers_each_state_element_once(dk, dv):
    g = geometry(dk, dv)
    RPL = g["RPL"]
    NB, EPB = (1, 2) if RPL == 2 else (RPL // 4, 4)
    seen = {}
    for warp in range(g["NWH"]):              # the warps of one v-head
        for lane in range(32):
            rg, cg = lane >> 2, lane & 3
            col = 16 * warp + 4 * cg
            for j, e in itertools.product(range(NB), range(EPB)):
                row = 2 * rg + e if RPL == 2 else 32 * j + 4 * rg + e
                for c in range(4):
                    seen[(row, col + c)] = seen.get((row, col + c), 0) + 1
    assert len(seen) == dk * dv and set(seen.values()) == {1}


@pytest.mark.parametrize("Hk,G,dk,dv", [(2, 1, 16, 32), (16, 2, 128, 128), (1, 8, 64, 16), (2, 3, 32, 64)])
def test_spec_commit_rolls_every_channel_of_a_sequence_exactly_once(Hk, G, dk, dv):
    # the commit kernel's channel map (csrc/gdn_spec.cu): the CTA of v-head h rolls its v
    # channels, and the k-head's q and k channels when h is the group's first v-head
    Hv = Hk * G
    C = 2 * Hk * dk + Hv * dv
    seen = [0] * C
    for h in range(Hv):
        hk = h // G
        nqk = 2 * dk if h % G == 0 else 0
        for i in range(nqk + dv):
            ch = 2 * Hk * dk + h * dv + (i - nqk) if i >= nqk else (hk * dk + i if i < dk else Hk * dk + hk * dk + (i - dk))
            seen[ch] += 1
    assert seen == [1] * C


@pytest.mark.parametrize("dk,dv", list(itertools.product((16, 32, 64, 128), (16, 32, 64, 128))))
def test_spec_commit_tile_covers_each_state_element_once(dk, dv):
    # the commit kernel's geometry (csrc/gdn_spec.cu, CommitGeo): thread -> RPT consecutive
    # rows x 4 columns of the dk x dv tile, NT = clamp(dk*dv/32, 32, 512) threads
    TPR = dv // 4
    NT = min(512, max(32, dk * dv // 32))
    RPP = NT // TPR
    RPT = dk // RPP
    assert NT % TPR == 0 and dk % RPP == 0 and RPT >= 1
    seen = {}
    for tid in range(NT):
        cg, row0 = tid % TPR, (tid // TPR) * RPT
        for r in range(RPT):
            for c in range(4):
                seen[(row0 + r, 4 * cg + c)] = seen.get((row0 + r, 4 * cg + c), 0) + 1
    assert len(seen) == dk * dv and set(seen.values()) == {1}

