"""Helpers shared by the GPU tests: host<->device moves of bf16 bit arrays and
the attention tolerance check (max-abs <= 1e-2 and relative L2 <= 5e-3, the
bound the target states for bf16 operands with fp32 accumulation)."""
import numpy as np

MAX_ABS = 1e-2
REL_L2 = 5e-3


def to_dev(bits: np.ndarray):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.cuda()


def dev_to_f64(t) -> np.ndarray:
    import torch
    return t.detach().view(torch.int16).cpu().numpy().view(np.uint16).astype(np.uint32).__lshift__(16) \
        .view(np.float32).astype(np.float64)


def attn_errors(got: np.ndarray, ref: np.ndarray):
    max_abs = float(np.max(np.abs(got - ref))) if got.size else 0.0
    rel = float(np.linalg.norm((got - ref).ravel()) / max(np.linalg.norm(ref.ravel()), 1e-300))
    return max_abs, rel


def assert_attn_close(got: np.ndarray, ref: np.ndarray, what: str = ""):
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    max_abs, rel = attn_errors(got, ref)
    assert max_abs <= MAX_ABS and rel <= REL_L2, f"{what}: max_abs={max_abs:.3e} rel_l2={rel:.3e}"
    return max_abs, rel


def sample_rows(Tq: int, n: int, seed: int) -> np.ndarray:
    """Rows 0 and Tq-1, every row of the last (partial) 128-row tile, and random rows."""
    rng = np.random.default_rng(seed)
    last_tile = np.arange((Tq - 1) // 128 * 128, Tq)
    rows = set([0, Tq - 1]) | set(last_tile.tolist()) | set(rng.choice(Tq, size=min(n, Tq), replace=False).tolist())
    return np.array(sorted(rows))


def assert_attn_close_derived(got: np.ndarray, ref: np.ndarray, vmax: float, what: str = ""):
    """Bound derived from the arithmetic for inputs whose softmax is peaked (a few
    keys dominate, |out| approaches max|v|). bf16 keeps 8 significant bits, so
    its unit roundoff is u = 2^-8: probabilities rounded to bf16 move the
    output by at most u * max|v| (each weight off by at most u relative, the
    weights sum to one), rounding the output to bf16 adds at most u * |out|;
    fp32 accumulation and exp2 add far less (1e-3 margin).
    The relative L2 bound stays the standard 5e-3."""
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    bound = 2.0 ** -8 * (vmax + np.abs(ref)) + 1e-3
    err = np.abs(got - ref)
    _, rel = attn_errors(got, ref)
    assert np.all(err <= bound) and rel <= REL_L2, \
        f"{what}: worst excess {float(np.max(err - bound)):.3e} rel_l2={rel:.3e}"
