"""Host-side checks of the chunked tensor-core multi-token kernel (csrc/gdn_decode_chunk.cu),
so that a change which breaks its index arithmetic or its pipeline fails here, before any
GPU run.

The kernel's compile-time constants (tile sizes, shared-memory offsets, TMEM columns) are
read from its source; the thread-to-data maps, the swizzled operand writes, the staged
copies and the barrier protocol are restated from the kernel and must be kept in step
with it. Checked:
  * the shared-memory layout: alignment of every region the tensor core, the bulk copies
    and the vector loads touch, no overlap, the 227 KB limit;
  * the operand tiles: the producers' writes, read back through the 128-byte swizzle as
    the tensor core reads a K-major operand from a shared-memory descriptor, give each
    MMA exactly the rows and K slice it multiplies;
  * the TMEM column plan and every thread map (each element written once);
  * every cp.async of the staging stays inside its source tensor and its destination
    region, 16-byte aligned, for all conv widths and token counts;
  * the barrier protocol between producers, consumers, the bulk copies and the MMAs,
    run under randomised schedules: no deadlock, no buffer overwritten before it is read,
    every read sees the data meant for it, every unit's output and state written once."""
import collections
import itertools
import pathlib
import random
import re

import pytest

CSRC = pathlib.Path(__file__).resolve().parents[1] / "gated_delta_rule_102_b200" / "csrc"
SMEM_LIMIT = 232448  # dynamic shared memory one CTA may use (227 KB)


def kernel_constants():
    """The namespace-scope constexpr integers of the kernel's source, evaluated in order."""
    env = {}
    m = re.search(r"constexpr int kMaxConvWidth = (\d+);", (CSRC / "gdn_device.cuh").read_text())
    env["kMaxConvWidth"] = int(m.group(1))
    for line in (CSRC / "gdn_decode_chunk.cu").read_text().splitlines():
        m = re.match(r"constexpr (?:int|uint32_t) ([^;]*);", line)  # (not indented: namespace scope)
        if not m:
            continue
        for decl in m.group(1).split(","):
            name, expr = decl.split("=", 1)
            env[name.strip()] = eval(expr.replace("/", "//"), {}, env)  # integer arithmetic only
    return env


K = kernel_constants()


def test_constants_were_read():
    for name in ("kCT", "kDK", "kDV", "kProducers", "kXRegion", "kXBuf", "kZBuf", "kHeadFloats", "OFF_HEAD",
                 "kSmemBytes", "TM_AHI", "TM_ALO", "TM_D2", "TM_D1", "TM_D1B", "TM_YHI", "TM_YLO", "kTmemCols"):
        assert name in K, name
    # the maps below assume these sizes (two producer threads per q|k channel pair, and so on)
    assert (K["kCT"], K["kDK"], K["kDV"], K["kProducers"], K["kRing"], K["kChunksPerTile"]) == (16, 128, 128, 256, 4, 4)


# ---------------------------------------------------------------- shared memory

def regions():
    """name -> (byte offset from the 1024-byte aligned base, size)"""
    ct, dk, dv = K["kCT"], K["kDK"], K["kDV"]
    return {
        "ring": (K["OFF_RING"], K["kRing"] * K["kChunkBytes"]),
        "x": (K["OFF_X"], 2 * K["kXBuf"]),
        "z": (K["OFF_Z"], 2 * K["kZBuf"]),
        "gram": (K["OFF_GRAM"], 2 * 2 * ct * ct * 4),
        "scratch": (K["OFF_SCR"], ct * K["kScrStride"] * 4),
        "graw": (K["OFF_GRAW"], K["kGroupRawBytes"]),
        "norms": (K["OFF_NRM"], 2 * ct * 4),
        "heads": (K["OFF_HEAD"], 2 * K["kHeadFloats"] * 4),
        "barriers": (K["OFF_BAR"], K["kNumBars"] * 8),
        "misc": (K["OFF_MISC"], 16),
    }


def test_shared_memory_regions_are_disjoint_aligned_and_fit():
    r = sorted(regions().items(), key=lambda kv: kv[1][0])
    for (na, (oa, sa)), (nb, (ob, _)) in zip(r, r[1:]):
        assert oa + sa <= ob, (na, nb)
    last, (o, s) = r[-1]
    assert o + s + 1024 <= K["kSmemBytes"] <= SMEM_LIMIT  # + the slack that aligns the base
    # swizzled operand tiles: 1024-byte atoms; the bulk copies and cp.async: 16 bytes;
    # mbarriers: 8 bytes
    for name in ("x", "z"):
        assert regions()[name][0] % 1024 == 0
    assert K["kXRegion"] % 1024 == 0 and K["kXBuf"] % 1024 == 0 and K["kZBuf"] % 1024 == 0
    assert K["OFF_RING"] % 16 == 0 and K["kChunkBytes"] % 16 == 0
    for name in ("scratch", "graw", "heads"):
        assert regions()[name][0] % 16 == 0, name
    assert K["OFF_BAR"] % 8 == 0
    assert K["kNumBars"] == K["kRing"] + 2 * 4 + 2  # ring, group/unit full/empty, update and first GEMM


def test_unit_buffer_layout():
    """One unit buffer: v [16][128] f32 (o once solved), alpha, beta, gamma, w [16], A and M
    [16][16], z [16][128] bf16, then 4 ints (first row, head, count)."""
    ct, dv = K["kCT"], K["kDV"]
    fields = [("v", ct * dv * 4), ("alpha", ct * 4), ("beta", ct * 4), ("gamma", ct * 4), ("w", ct * 4),
              ("A", ct * ct * 4), ("M", ct * ct * 4), ("z", ct * dv * 2), ("meta", 16)]
    off, at = 0, {}
    for name, size in fields:
        at[name] = off
        off += size
    assert off == K["kHeadFloats"] * 4
    # float4 reads of v/o rows, beta, gamma and the coefficient rows; uint2 reads and 16-byte
    # cp.async of z; int meta
    for name in ("v", "beta", "gamma", "A", "M", "z"):
        assert at[name] % 16 == 0, name
    assert (K["kHeadFloats"] * 4) % 16 == 0  # the second buffer too
    assert at["meta"] == (K["kHeadFloats"] - 4) * 4


def test_unit_staging_fits_in_the_scratch_and_misses_the_group_staging():
    # the unit phase stages its v rows in the scratch's place, while the next group's q|k rows
    # may be landing in graw
    scr_off, scr_size = regions()["scratch"]
    graw_off, _ = regions()["graw"]
    assert K["kUnitRawBytes"] <= scr_size and scr_off + K["kUnitRawBytes"] <= graw_off
    assert K["kScrStride"] * 4 % 16 == 0 and K["kScrStride"] >= 2 * K["kDK"]  # float4 rows of raw q | raw k


# ---------------------------------------------------------------- operand tiles

def sw128(addr):
    """The 128-byte swizzle of a 1024-byte aligned tile: the 16-byte chunk index (address
    bits 4..6) XORed with the row within the 8-row atom (bits 7..9)."""
    return addr ^ (((addr >> 7) & 7) << 4)


def kmajor_read(start, row, k):
    """Byte address of element (row, k) of a tf32 operand as the tensor core reads it from a
    K-major descriptor with the 128-byte swizzle: 128-byte rows, 8-row atoms 1024 bytes
    apart (the stride byte offset), K advanced by moving the start address."""
    return sw128(start + (row // 8) * 1024 + (row % 8) * 128 + 4 * k)


def x_tile_writes(gb):
    """byte offset in the X buffers -> (part, row, dk) for every element the producers
    write: thread i, row = i / 8, 16-byte groups j = i % 8 + 8 m; high parts in rows 0..31,
    low parts 32 rows (4 KiB) further."""
    out = {}
    for i in range(K["kProducers"]):
        row = i >> 3
        for m in range(4):
            j = (i & 7) + 8 * m
            off = gb * K["kXBuf"] + (j >> 3) * K["kXRegion"] + row * 128 + (((j & 7) ^ (row & 7)) << 4)
            for e in range(4):
                for part, base in (("hi", 0), ("lo", 32 * 128)):
                    a = off + base + 4 * e
                    assert a not in out
                    out[a] = (part, row, 4 * j + e)
    return out


@pytest.mark.parametrize("gb", [0, 1])
def test_operand_tile_is_what_the_first_gemm_reads(gb):
    w = x_tile_writes(gb)
    assert len(w) == 64 * K["kDK"]  # [k | q] x dk, high and low: every element once
    assert min(w) >= gb * K["kXBuf"] and max(w) < (gb + 1) * K["kXBuf"]
    # chunk q of the state tile: 4 MMAs of K = 8 from the descriptor of region q, start + 32 kk
    # bytes; N = 64 reads rows 0..63 (high then low), N = 32 rows 0..31 (high)
    for q in range(K["kChunksPerTile"]):
        for kk in range(4):
            start = gb * K["kXBuf"] + q * K["kXRegion"] + 32 * kk
            for n in range(64):
                for k in range(8):
                    part, row = ("hi", n) if n < 32 else ("lo", n - 32)
                    assert w[kmajor_read(start, n, k)] == (part, row, 32 * q + 8 * kk + k)


def z_tile_writes(gb):
    """byte offset in the Z buffers -> (part, dk row, token): thread i takes row i % 128 and
    token quads 2 (i / 128) and 2 (i / 128) + 1, high parts in the first 64 bytes of the row."""
    out = {}
    for i in range(K["kProducers"]):
        zrow = i & (K["kDK"] - 1)
        for jj in range(2):
            j = 2 * (i // K["kDK"]) + jj
            for e in range(4):
                for part, chunk in (("hi", j), ("lo", j + 4)):
                    a = gb * K["kZBuf"] + zrow * 128 + ((chunk ^ (zrow & 7)) << 4) + 4 * e
                    assert a not in out
                    out[a] = (part, zrow, 4 * j + e)
    return out


@pytest.mark.parametrize("gb", [0, 1])
def test_key_tile_is_what_the_update_gemm_reads(gb):
    w = z_tile_writes(gb)
    assert len(w) == 2 * K["kDK"] * K["kCT"]
    assert min(w) >= gb * K["kZBuf"] and max(w) < (gb + 1) * K["kZBuf"]
    # the update: N = dk rows, 8 tokens per MMA; high parts from start + 32 kk, low parts from
    # start + 32 (kk + 2)
    for kk in range(K["kCT"] // 8):
        for part, start in (("hi", 32 * kk), ("lo", 32 * (kk + 2))):
            for r in range(K["kDK"]):
                for k in range(8):
                    assert w[kmajor_read(gb * K["kZBuf"] + start, r, k)] == (part, r, 8 * kk + k)


def test_tmem_column_plan():
    """Each accumulator and TMEM operand in its own columns, all inside the allocation."""
    ct, dk = K["kCT"], K["kDK"]
    spans = {
        "S0 high (A of the first GEMM)": (K["TM_AHI"], dk),
        "S0 low (A of the first GEMM)": (K["TM_ALO"], dk),
        "update accumulator (N = dk)": (K["TM_D2"], dk),
        "first GEMM, high S0 (N = 64)": (K["TM_D1"], 4 * ct),
        "first GEMM, low S0 (N = 32)": (K["TM_D1B"], 2 * ct),
        "w delta high (A of the update)": (K["TM_YHI"], ct),
        "w delta low (A of the update)": (K["TM_YLO"], ct),
    }
    cols = [None] * K["kTmemCols"]
    for name, (c0, n) in spans.items():
        assert c0 + n <= K["kTmemCols"], name
        for c in range(c0, c0 + n):
            assert cols[c] is None, (name, cols[c])
            cols[c] = name
    n = K["kTmemCols"]
    assert n >= 32 and n & (n - 1) == 0 and n <= 512  # an allocation is a power of two, 32..512 columns
    # the first GEMM's A slices (32 q + 8 kk, 8 columns) and the partial-sum loads (16 columns)
    for q, kk in itertools.product(range(4), range(4)):
        assert 32 * q + 8 * kk + 8 <= dk
    for which, h16 in itertools.product(range(3), range(2)):
        base = (K["TM_D1"], K["TM_D1"] + 2 * ct, K["TM_D1B"])[which] + 16 * h16
        assert spans["first GEMM, high S0 (N = 64)"][0] <= base and base + 16 <= K["TM_D1B"] + 2 * ct


# ---------------------------------------------------------------- thread maps

def test_thread_maps_cover_each_element_once():
    ct, dk, dv, npr = K["kCT"], K["kDK"], K["kDV"], K["kProducers"]
    pw_count = npr // 32
    # q|k conv: producer i owns channel i (all tokens)
    assert npr == 2 * dk
    # v conv: producer i owns channel i % dv for the tokens 8 (i / dv) .. 8 (i / dv) + 7
    half = ct // 2
    cover = collections.Counter((i % dv, (i // dv) * half + t) for i in range(npr) for t in range(half))
    assert cover == collections.Counter(itertools.product(range(dv), range(ct)))
    # the gates of token gi on lanes 0..15 of the last producer warp (they prefetch its inputs too)
    gates = [i - (npr - 32) for i in range(npr) if 0 <= i - (npr - 32) < ct]
    assert gates == list(range(ct))
    # norms: warp pw takes tokens pw + 8 m
    assert sorted(pw + pw_count * m for pw in range(pw_count) for m in range(ct // pw_count)) == list(range(ct))
    # Gram products and solve coefficients: thread i one (t, s)
    assert sorted((i >> 4, i & 15) for i in range(npr)) == list(itertools.product(range(ct), range(ct)))
    # the gated RMSNorm: warp pw takes tokens pw, pw + 8, ...; lane l columns 4 l .. 4 l + 3
    toks = collections.Counter(t for pw in range(pw_count) for t in range(pw, ct, pw_count))
    assert toks == collections.Counter(range(ct))
    assert sorted(4 * l + e for l in range(32) for e in range(4)) == list(range(dv))
    # consumers: thread c (column c) loads chunk q's rows 16 hh + r and stores rows 32 q + r
    loaded = sorted(32 * q + 16 * hh + r for q in range(4) for hh in range(2) for r in range(16))
    stored = sorted(32 * q + r for q in range(4) for r in range(32))
    assert loaded == stored == list(range(dk))
    assert K["kConsumerWarps"] * 32 == dv  # one consumer thread (and TMEM lane) per column


# ---------------------------------------------------------------- staged copies

@pytest.mark.parametrize("W", range(1, K["kMaxConvWidth"] + 1))
@pytest.mark.parametrize("Hk,G", [(1, 1), (2, 4), (3, 2), (16, 2)])
def test_staged_copies_stay_in_bounds(W, Hk, G):
    ct, dk, dv = K["kCT"], K["kDK"], K["kDV"]
    Hv = Hk * G
    C = 2 * Hk * dk + Hv * dv
    assert C % 8 == 0  # every row of qkv and of a conv slot starts 16-byte aligned
    graw_elems = K["kGroupRawBytes"] // 2
    gwt = K["kRawRows"] * 2 * dk
    uw = K["kRawRows"] * dv
    for n in range(0, ct + 1):
        nr = W - 1 + n
        assert nr <= K["kRawRows"]
        for kh in range(Hk):
            # the group's q and k rows: 16-byte pieces, two runs of 128 channels per row
            for e in range(0, nr * 32):
                r, part, off = e >> 5, (e >> 4) & 1, (e & 15) * 8
                dst = r * 2 * dk + part * dk + off
                assert dst % 8 == 0 and dst + 8 <= gwt
                ch = (part * Hk + kh) * dk + off
                assert ch % 8 == 0 and ch + 8 <= 2 * Hk * dk  # inside the q|k channels
                if r < W - 1:
                    assert r * C + ch + 8 <= (W - 1) * C  # inside the slot's history
                else:
                    assert r - (W - 1) < n  # one of the sequence's tokens
            wpieces = dk * W // 8
            for e in range(2 * wpieces):
                part = int(e >= wpieces)
                o = e - part * wpieces
                dst = gwt + part * dk * W + o * 8
                assert dst % 8 == 0 and dst + 8 <= graw_elems
                src = (part * Hk + kh) * dk * W + o * 8
                assert src % 8 == 0 and src + 8 <= 2 * Hk * dk * W
        for hh in range(Hv):
            cv = 2 * Hk * dk + hh * dv
            for e in range(nr * 16):
                r, off = e >> 4, (e & 15) * 8
                assert r * dv + off + 8 <= uw and (cv + off) % 8 == 0 and cv + off + 8 <= C
            for e in range(dv * W // 8):
                assert uw + e * 8 + 8 <= K["kUnitRawBytes"] // 2
                assert (cv * W + e * 8) % 8 == 0 and cv * W + e * 8 + 8 <= C * W
            for e in range(n * 16):  # z rows into the unit buffer: [16][128] bf16
                t, off = e >> 4, (e & 15) * 8
                assert t * dv + off + 8 <= ct * dv
