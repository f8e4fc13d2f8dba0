"""The append/recache kernel's work split, restated on the CPU.

The kernel (kv_scatter.cuh) cuts the source rows ((token, head) pairs) of every
source layer and frame into units of kRows rows, never across a frame, and
gives CTA c of G the units [U*c/G, U*(c+1)/G). Each unit is one bulk copy of
K rows and one of V rows into a stage of shared memory, and each CTA counts
its units of every layer it touches into that layer's completion word. This
restatement checks, for many geometries and both unit sizes, that every
source row is copied exactly once, that every copy and shared-memory access
stays inside its buffer, and that the completion counts of a layer add up to
its unit count (so exactly one CTA advances the counters). The constants below
are the kernel's (ScatterTile in kv_scatter.cuh)."""
import pytest

THREADS_CONSUMER = 256
UNIT_PASS_BYTES = 8192            # one pass: 256 / (D/16) rows of D bf16 values
SMEM_LIMIT = 227 * 1024


def tile(D: int, passes: int):
    lpr = D // 16
    pass_rows = THREADS_CONSUMER // lpr
    rows = passes * pass_rows
    row_bytes = 2 * D
    unit_bytes = rows * row_bytes
    stages = 2 if passes == 2 else 6
    ctas_per_sm = 3 if passes == 2 else 2
    smem = stages * 2 * unit_bytes + stages * (8 + 8 + 16) + 16 + 512
    return dict(lpr=lpr, pass_rows=pass_rows, rows=rows, row_bytes=row_bytes, unit_bytes=unit_bytes,
                stages=stages, ctas_per_sm=ctas_per_sm, smem=smem)


def check_partition(L, H, D, T, n_layers, n_frames, slot_frames, passes, sms=148, round_up=True):
    c = tile(D, passes)
    assert c["unit_bytes"] == passes * UNIT_PASS_BYTES
    # two (recache: three) CTAs of this size must fit one SM's shared memory
    assert c["smem"] <= SMEM_LIMIT and c["ctas_per_sm"] * (c["smem"] + 1024) <= 228 * 1024
    rows_frame = T * H
    per_frame = -(-rows_frame // c["rows"]) if round_up else rows_frame // c["rows"]
    per_layer = n_frames * per_frame
    n_units = n_layers * per_layer
    grid = min(n_units, sms * c["ctas_per_sm"])
    src_rows = n_layers * n_frames * rows_frame
    slots = slot_frames * T
    planes = L * 2 * H
    copied = bytearray(src_rows)
    counted = [0] * n_layers
    for cta in range(grid):
        u0, u1 = n_units * cta // grid, n_units * (cta + 1) // grid
        assert u1 > u0, "every CTA owns a unit"
        cur = -1
        for u in range(u0, u1):
            li, rem = divmod(u, per_layer)
            fi, b = divmod(rem, per_frame)
            if li != cur:                      # the CTA enters a layer: it counts its units there once
                cur = li
                counted[li] += min(u1, (li + 1) * per_layer) - u
            row0 = b * c["rows"]
            nrows = min(c["rows"], rows_frame - row0)
            srow = (li * n_frames + fi) * rows_frame + row0
            nbytes = nrows * c["row_bytes"]
            assert nrows > 0 and 0 <= srow and srow + nrows <= src_rows
            assert (srow * c["row_bytes"]) % 16 == 0 and nbytes % 16 == 0 and nbytes <= c["unit_bytes"]
            for r in range(c["rows"]):         # consumer reads: inside the unit's stage
                assert r * c["row_bytes"] + 32 * (c["lpr"] - 1) + 32 <= c["unit_bytes"]
            for r in range(nrows):
                copied[srow + r] += 1
                t, hh = divmod(row0 + r, H)
                assert t < T
                for slot in (0, slot_frames - 1):
                    assert slot * T + t < slots
                for kv in (0, 1):
                    assert (li * 2 + kv) * H + hh < planes
    assert all(x == 1 for x in copied), "every source row is copied exactly once"
    assert counted == [per_layer] * n_layers, "the completion counts of each layer reach its unit count"


CASES = [
    # L, H, D, T, source layers, frames per source layer, frame slots per plane
    (30, 12, 128, 1560, 1, 3, 12),      # Wan-1.3B append of one layer
    (30, 12, 128, 1560, 30, 3, 12),     # all layers in one launch
    (2, 12, 128, 1560, 2, 12, 12),      # recache of a 2-layer stack
    (2, 2, 64, 16, 2, 3, 9),
    (1, 3, 128, 7, 1, 3, 12),
    (2, 1, 64, 5, 2, 3, 3),
    (1, 2, 128, 4, 1, 2, 4),
    (1, 2, 64, 3, 1, 2, 3),
    (1, 1, 128, 2, 1, 1, 5),
    (3, 2, 128, 20, 3, 3, 7),
    (1, 5, 64, 33, 1, 9, 12),
    (4, 7, 64, 129, 4, 2, 6),           # rows per frame not a multiple of any unit
]


@pytest.mark.parametrize("passes", [1, 2])
@pytest.mark.parametrize("L,H,D,T,n_layers,n_frames,slot_frames", CASES)
def test_scatter_units_cover_every_row_once_inside_the_buffers(L, H, D, T, n_layers, n_frames, slot_frames,
                                                                passes):
    check_partition(L, H, D, T, n_layers, n_frames, slot_frames, passes)


def test_partition_check_catches_a_dropped_tail():
    """A plausible mistake, a unit count per frame that rounds the frame's rows
    down, leaves each frame's tail rows uncopied; the check must fail on it."""
    with pytest.raises(AssertionError, match="exactly once"):
        check_partition(1, 12, 128, 7, 1, 3, 12, 1, round_up=False)
