"""Launch geometry of the two attention kernels, checked on the CPU for every workload shape
and every shape the GPU tests and the timing probe use.

The host's split choice and the kernels' index arithmetic are replayed here, and each
TMA coordinate, shared-memory offset, TMEM column and output index is checked against
the buffer or tensor map it addresses:
- TMA x coordinates are multiples of 16 bytes, and every box starts inside its tensor;
- the low-term window (the call's own K/V low parts, rows counted from `base`) fits the
  workspace's window of lo_rows rows;
- slots and query tiles stay inside the kernel's shared memory, TMEM columns below 512;
- heads stay inside one KV head's group, and every output and partial index stays
  inside its buffer (partials: at most 16 splits of [nq][rows][128] fp32).
Both kernels' half-slot plans are also checked against the barrier simulation's.
"""

import pytest

from block_diffusion_lm_masked_b200 import configs as CF

NUM_SMS = 148
MAX_SPLITS = 16
D = 128


def cdiv(a, b):
    return -(-a // b)


def lo_rows(T):
    return cdiv(T, 128) * 128 + 128


def splits_single(n_q, nq, n_keys):
    nch = cdiv(n_keys, 128)
    s = NUM_SMS // (cdiv(n_q, 128) * nq)
    s = max(min(s, MAX_SPLITS, nch // 2), 1)
    cps = cdiv(nch, s)
    return cdiv(nch, cps), cps


def head_groups(nq, group, pair=True):
    return nq // 2 if (pair and group % 2 == 0) else nq


def splits_pair(n_q, nq, group, n_keys, pair=True):
    nch = cdiv(n_keys, 128)
    s = NUM_SMS // (cdiv(n_q, 128) * head_groups(nq, group, pair))
    s = max(min(s, MAX_SPLITS, nch // 2), 1)
    cps = cdiv(nch, s)
    return cdiv(nch, cps), cps


def choose_pair(n_q, nq, group, n_keys):
    """The host's choice for the head-pair kernel: pairs unless single heads fill at least
    a quarter more SMs in the one wave.  Returns (pair, splits, chunks per split)."""
    sp_p, cps_p = splits_pair(n_q, nq, group, n_keys, True)
    sp_s, cps_s = splits_pair(n_q, nq, group, n_keys, False)
    tiles = cdiv(n_q, 128)
    pair = group % 2 == 0 and 4 * (tiles * nq * sp_s) < 5 * (tiles * head_groups(nq, group, True) * sp_p)
    return (pair, sp_p, cps_p) if pair else (False, sp_s, cps_s)


def debug_entry_accepts(n_q, pos0, n_keys, causal, cap, nq, nkv):
    """The debug entries' host checks (dg_debug_attention_bf16 / _pair_bf16)."""
    if not (nq > 0 and nkv > 0 and nq % nkv == 0 and n_q > 0 and n_keys > 0 and n_keys <= cap and cap % 8 == 0):
        return False
    if causal and pos0 + n_q > n_keys:
        return False
    if pos0 < 0 or pos0 > n_keys:
        return False
    return n_keys - (pos0 // 128) * 128 <= lo_rows(n_q)


class HalfSlotPlan:
    """The head-pair kernel's half-slot ring: ring entries taken in plan order (a chunk's K
    parts, then its V^T parts, two each for own keys), entry e in half-slot e % slots as
    that half-slot's use e // slots (a2_slot and the use parity in the kernel)."""

    def __init__(self, slots=3):
        self.nxt, self.uses, self.slots = 0, [0] * slots, slots

    def take(self, cur):
        k, v = [], []
        for lst in (k, v):
            for _ in range(2 if cur else 1):
                lst.append((self.nxt, self.uses[self.nxt]))
                self.uses[self.nxt] += 1
                self.nxt = (self.nxt + 1) % self.slots
        return k, v


class TwoRingPlan:
    """The single-head kernel's rings: a chunk's K parts take the next entries of a ring of
    kslots half-slots, its V^T parts those of a ring of vslots half-slots numbered after
    the K ring's (at_kslot / at_vslot and the use parities in the kernel)."""

    def __init__(self, kslots=3, vslots=2):
        self.ek = self.ev = 0
        self.kslots, self.vslots = kslots, vslots

    def take(self, cur):
        n = 2 if cur else 1
        k = [((self.ek + i) % self.kslots, (self.ek + i) // self.kslots) for i in range(n)]
        v = [(self.kslots + (self.ev + i) % self.vslots, (self.ev + i) // self.vslots) for i in range(n)]
        self.ek += n
        self.ev += n
        return k, v


def check_tma(x, y, elem_bytes, y_extent):
    assert (x * elem_bytes) % 16 == 0, f"TMA x {x} not 16-byte aligned"
    assert 0 <= y < y_extent, f"box starts outside the tensor (row {y} of {y_extent})"


def audit(kernel, n_q, pos0, n_keys, causal, nq, nkv, T):
    """Every CTA of one attention launch; T: the workspace's token capacity (>= n_q)."""
    assert T >= n_q
    group = nq // nkv
    base = (pos0 // 128) * 128
    Lc = lo_rows(T)
    assert 0 <= n_keys - base <= Lc, "the low-term window exceeds the workspace's"
    W = 128
    if kernel == "pair":
        pair, n_splits, cps = choose_pair(n_q, nq, group, n_keys)
        nh = 2 if pair else 1
        ys = head_groups(nq, group, pair)
        smem_q, slot_bytes, slots = 2 * 4 * 16384, 32768, 3      # half-slots of 32 KB
        smem_total = 1024 + smem_q + slots * slot_bytes
        assert smem_total <= 227 * 1024 - 512
    else:
        n_splits, cps = splits_single(n_q, nq, n_keys)
        nh, ys = 1, nq
        smem_q, slot_bytes, slots = 4 * 16384, 32768, 5         # the query tile, 3 + 2 half-slots
        smem_total = 1024 + smem_q + slots * slot_bytes
        assert smem_total <= 227 * 1024 - 512
        # TMEM columns: S buffers 0..127 and 128..255, O 256..383, P buffers 384..447 and 448..511
        cols = [(0, 128), (128, 128), (256, 128), (384, 64), (448, 64)]
        assert sorted(cols) == cols and all(a + n <= b for (a, n), (b, _) in zip(cols, cols[1:]))
        assert cols[-1][0] + cols[-1][1] <= 512
    assert 1 <= n_splits <= MAX_SPLITS
    part_o_len = MAX_SPLITS * nq * T * D
    out_len = n_q * nq * D
    chunks_seen = 0
    for qt in range(cdiv(n_q, 128)):
        q_row0 = qt * 128
        rows_here = min(128, n_q - q_row0)
        kv_end = min(n_keys, pos0 + q_row0 + rows_here) if causal else n_keys
        nch_total = cdiv(kv_end, W)
        for y in range(ys):
            h0 = y * nh
            kvh = h0 // group
            assert kvh < nkv and h0 + nh <= nq
            assert all((h0 + i) // group == kvh for i in range(nh)), "a CTA's heads span two KV heads"
            for hl in range(nh):  # the query tiles (hi and lo maps: x = d 0 / 64, y = row, z = head)
                assert h0 + hl < nq
                check_tma(0, q_row0, 2, n_q)
                check_tma(64, q_row0, 2, n_q)
            for sp in range(n_splits):
                c_begin = sp * cps
                nck = min(nch_total, c_begin + cps) - c_begin
                rows = [q_row0 + r for r in range(128) if q_row0 + r < n_q]
                if nck <= 0:
                    for h in range(h0, h0 + nh):
                        for r in rows:
                            assert ((sp * nq + h) * n_q + r + 1) * D <= part_o_len
                    continue
                plan = HalfSlotPlan(slots) if kernel == "pair" else TwoRingPlan()
                for j in range(nck):
                    key0 = (c_begin + j) * W
                    assert key0 < kv_end
                    cur = key0 >= base
                    k_parts, v_parts = plan.take(cur)
                    for i, ((sk, _), (sv, _)) in enumerate(zip(k_parts, v_parts)):
                        krow = key0 if i == 0 else key0 - base
                        extent = n_keys if i == 0 else n_keys - base
                        assert krow % W == 0 and krow < extent
                        check_tma(0, krow, 2, extent)       # K blocks: x = d 0 / 64, y = key row
                        check_tma(64, krow, 2, extent)
                        check_tma(krow, 0, 2, extent + 1)   # V^T blocks: x = key, key + 64; y = d 0
                        check_tma(krow + 64, 0, 2, extent + 64)
                        for hs in (sk, sv):
                            assert hs < slots and smem_q + (hs + 1) * slot_bytes <= smem_total - 1024
                    chunks_seen += 1
                if kernel == "pair":
                    for hl in range(nh):
                        assert hl * 256 + 128 <= 512           # S/P region: S 128 fp32, P hi 64 + lo 64
                        assert hl * 256 + 128 + 128 <= 512     # O
                for h in range(h0, h0 + nh):
                    for r in (rows[0], rows[-1]):
                        if n_splits == 1:
                            assert r * nq * D + h * D + D <= out_len
                        else:
                            assert ((sp * nq + h) * n_q + r + 1) * D <= part_o_len
                            assert (sp * nq + h) * n_q + r < MAX_SPLITS * nq * T
    # every chunk of every tile is taken by exactly one split
    want = sum(cdiv(min(n_keys, pos0 + qt * 128 + min(128, n_q - qt * 128)) if causal else n_keys, W)
               for qt in range(cdiv(n_q, 128))) * ys
    assert chunks_seen == want
    return n_splits


def workload_launches():
    """(name, n_q, pos0, n_keys, causal, nq, nkv, T) of every attention launch the bf16
    workloads make: the denoising pass, and for the chained workload the prompt's prefill
    and each canvas's append."""
    out = []
    for name, c in CF.CONFIGS.items():
        if c["dtype"] != "bf16":
            continue
        nq, nkv, C = c["n_q_heads"], c["n_kv_heads"], c["canvas"]
        P = c.get("prefix", 0)
        if c.get("prompt"):
            pr = c["prompt"]
            out.append((name + ":prompt", pr, 0, pr, True, nq, nkv, max(pr, C)))
            for i in range(c.get("n_canvases", 1)):
                p0 = pr + i * C
                out.append((name + f":pass{i}", C, p0, p0 + C, False, nq, nkv, max(pr, C)))
                out.append((name + f":append{i}", C, p0, p0 + C, True, nq, nkv, max(pr, C)))
        else:
            out.append((name + ":pass", C, P, P + C, False, nq, nkv, C))
            out.append((name + ":append", C, P, P + C, True, nq, nkv, C))
    # the batched pass at its largest test batch runs each canvas's attention on a view
    # of a workspace sized for all B * C rows
    c = CF.CONFIGS["layer1_bf16"]
    out.append(("layer1_bf16:batched4", c["canvas"], c["prefix"], c["prefix"] + c["canvas"], False,
                c["n_q_heads"], c["n_kv_heads"], 4 * c["canvas"]))
    return out


DEBUG_SHAPES = [
    # nq, nkv, n_q, pos0, n_keys, causal: the GPU tests' and the probe's shapes
    (4, 2, 100, 200, 300, False), (16, 4, 256, 1024, 1280, False), (4, 1, 200, 50, 250, True),
    (2, 2, 64, 4900, 4964, False), (2, 1, 300, 0, 300, True), (8, 2, 256, 16128, 16384, False),
    (2, 1, 1024, 0, 1024, True), (16, 8, 256, 8192 - 256, 8192, False),
]


@pytest.mark.parametrize("kernel", ["single", "pair"])
@pytest.mark.parametrize("launch", workload_launches(), ids=lambda t: t[0])
def test_workload_launch_geometry(kernel, launch):
    _, n_q, pos0, n_keys, causal, nq, nkv, T = launch
    audit(kernel, n_q, pos0, n_keys, causal, nq, nkv, T)


@pytest.mark.parametrize("kernel", ["single", "pair"])
@pytest.mark.parametrize("shape", DEBUG_SHAPES)
def test_debug_shape_geometry(kernel, shape):
    nq, nkv, n_q, pos0, n_keys, causal = shape
    cap = cdiv(n_keys, 8) * 8 + 8
    assert debug_entry_accepts(n_q, pos0, n_keys, causal, cap, nq, nkv)
    audit(kernel, n_q, pos0, n_keys, causal, nq, nkv, n_q)


def test_every_accepted_debug_call_has_a_valid_geometry():
    """Sweep small shapes: whatever the debug entries accept launches within bounds."""
    n = 0
    for nq, nkv in ((2, 1), (2, 2), (4, 2), (6, 3), (8, 2)):
        for n_q in (1, 64, 129, 300):
            for n_keys in (1, 63, 64, 200, 511, 700):
                for pos0 in sorted({0, 1, n_keys - n_q, n_keys - n_q - 130, n_keys // 2, n_keys}):
                    for causal in (False, True):
                        cap = cdiv(n_keys, 8) * 8
                        if not debug_entry_accepts(n_q, pos0, n_keys, causal, cap, nq, nkv):
                            continue
                        for kernel in ("single", "pair"):
                            audit(kernel, n_q, pos0, n_keys, causal, nq, nkv, n_q)
                        n += 1
    assert n > 200


def test_debug_entries_refuse_a_low_term_window_past_the_workspace():
    """Queries far before the end of the keys would put the low-term window's tensor map
    past the workspace's window: the entries refuse that on the host."""
    import ctypes

    from block_diffusion_lm_masked_b200 import dg
    assert not debug_entry_accepts(64, 0, 4096, False, 4096, 2, 1)
    P = ctypes.c_void_p(256)
    for name in ("dg_debug_attention_bf16", "dg_debug_attention_pair_bf16"):
        f = getattr(dg.lib, name)
        assert f(P, P, P, 4096, 64, 0, 4096, 0, 2, 1, P, None, P, 1 << 30, None) == dg.DG_ERR_INVALID_ARG
        assert "window" in dg.lib.dg_last_error().decode()
        assert f(P, P, P, 4096, 64, -1, 4096, 0, 2, 1, P, None, P, 1 << 30, None) == dg.DG_ERR_INVALID_ARG
        assert f(P, P, P, 4096, 64, 4097, 4096, 0, 2, 1, P, None, P, 1 << 30, None) == dg.DG_ERR_INVALID_ARG


@pytest.mark.parametrize("slots", [2, 3])
def test_ring_arithmetic_counts_the_loads_of_each_half_slot(slots):
    """The wind-down's count of loads issued into each half-slot (a2_loads_into /
    at_loads_into) is the number of ring entries below the issued count in that half-slot,
    and the last one's use parity is what the drain waits for (rings of 3 in the head-pair
    kernel, of 3 and 2 in the single-head kernel)."""
    def loads_into(s, n):
        return (n - 1 - s) // slots + 1 if n > s else 0
    for n in range(0, 40):
        for s in range(slots):
            mine = [e for e in range(n) if e % slots == s]
            assert loads_into(s, n) == len(mine)
            if mine:
                assert (loads_into(s, n) - 1) & 1 == (mine[-1] // slots) & 1


@pytest.mark.parametrize("nck,cur_from", [(5, 2), (9, 0), (12, 8), (3, 3)])
def test_kernel_slot_plans_are_the_simulated_ones(nck, cur_from):
    import test_pipeline_protocol as TP
    plan = HalfSlotPlan(3)
    got = [plan.take(j >= cur_from) for j in range(nck)]
    assert got == [(list(k), list(v)) for k, v in TP.half_slot_plan(nck, cur_from, 3)]
    plan2 = TwoRingPlan(3, 2)
    got2 = [plan2.take(j >= cur_from) for j in range(nck)]
    assert got2 == [(list(k), list(v)) for k, v in TP.two_ring_plan(nck, cur_from, 3, 2)]


def test_splits_fill_about_one_wave():
    """The head-pair kernel's launch stays within one wave of 148 SMs at the workload
    shapes (one CTA per SM: 225 KB of shared memory), and the pair / single-head choice
    takes the fuller wave: single heads at the single-layer size (128 CTAs against 80 in
    pairs), pairs at the large model (144 against 128)."""
    chosen = {}
    for name, c in CF.CONFIGS.items():
        if c["dtype"] != "bf16":
            continue
        nq, nkv, C, P = c["n_q_heads"], c["n_kv_heads"], c["canvas"], c.get("prefix", 0)
        pair, s, _ = choose_pair(C, nq, nq // nkv, P + C)
        ctas = cdiv(C, 128) * head_groups(nq, nq // nkv, pair) * s
        assert ctas <= NUM_SMS, (name, ctas)
        chosen[name] = (pair, ctas)
    assert chosen["layer1_bf16"] == (False, 128)
    assert chosen["large4_bf16"] == (True, 144)
