"""Helpers shared by the GPU parity tests (no arithmetic of the method here)."""
import numpy as np

# Parity bar for hidden states and logits: max|d| <= 3e-2 absolute AND
# max|d| / max|ref| <= 2e-2, against the oracle on the same bf16 weights.
ABS_TOL = 3e-2
REL_TOL = 2e-2


def max_err(got, ref):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.isfinite(got).all(), "non-finite values"
    d = float(np.max(np.abs(got - ref))) if got.size else 0.0
    m = float(np.max(np.abs(ref))) if ref.size else 0.0
    return d, (d / m if m > 0 else d)


def assert_parity(got, ref, abs_tol=ABS_TOL, rel_tol=REL_TOL, what=""):
    d, r = max_err(got, ref)
    assert d <= abs_tol and r <= rel_tol, f"{what}: max|d|={d:.3e} rel={r:.3e} (bar {abs_tol}, {rel_tol})"
    return d, r


def bits_to_f64(b):
    return (np.asarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def to_dev_bf16(a_bits, torch):
    """uint16 bf16 bits (numpy) -> torch.bfloat16 CUDA tensor with the same bits."""
    t = torch.from_numpy(np.ascontiguousarray(a_bits).view(np.int16)).cuda()
    return t.view(torch.bfloat16)


def from_dev_bf16(t):
    return t.view(__import__("torch").int16).cpu().numpy().view(np.uint16)


def build_paged(kc, vc, page, seed):
    """Scatter contiguous caches [B][ctx][nkv][d] (bf16 bits) into a shuffled page pool
    [n_pages][nkv][page][d] with block table [B][max_pages]. Returns (kpool, vpool, bt)."""
    B, ctx, nkv, d = kc.shape
    mp = (ctx + page - 1) // page
    n_pages = B * mp
    rng = np.random.default_rng(seed)
    perm = rng.permutation(n_pages).astype(np.int32)
    bt = perm.reshape(B, mp)
    kpool = np.zeros((n_pages, nkv, page, d), np.uint16)
    vpool = np.zeros((n_pages, nkv, page, d), np.uint16)
    for b in range(B):
        for j in range(mp):
            rows = slice(j * page, min(ctx, (j + 1) * page))
            n = rows.stop - rows.start
            kpool[bt[b, j], :, :n] = kc[b, rows].transpose(1, 0, 2)
            vpool[bt[b, j], :, :n] = vc[b, rows].transpose(1, 0, 2)
    return kpool, vpool, bt


def gather_paged(pool, bt, ctx):
    """Inverse of build_paged for one pool: [B][ctx][nkv][d]."""
    B, mp = bt.shape
    n_pages, nkv, page, d = pool.shape
    out = np.zeros((B, ctx, nkv, d), np.uint16)
    for b in range(B):
        for j in range(mp):
            rows = slice(j * page, min(ctx, (j + 1) * page))
            n = rows.stop - rows.start
            out[b, rows] = pool[bt[b, j], :, :n].transpose(1, 0, 2)
    return out


def perturb_inputs(weights):
    """The same weights with every embedding value moved by one bf16 ulp (its lowest mantissa
    bit flipped). fp32 accumulation makes a fraction of a percent of the bf16 roundings at every
    rounding point of every layer land one ulp from the fp64 oracle's; this input change is of
    the same order, so the oracle's response to it measures the noise floor of the problem."""
    out = dict(weights)
    out["embed"] = weights["embed"] ^ np.uint16(1)
    return out


def assert_within_conditioning(got, ref, ref_perturbed, factor=2.0, what=""):
    """Parity where the fixed bar is tighter than the problem's conditioning (a deep
    random-init stack moves its logits by percents when its inputs move by one bf16 ulp).
    Pass if the fixed bar holds, or if the error is within `factor` times the oracle's own
    response to the one-ulp input change on the same input."""
    d, r = max_err(got, ref)
    floor = float(np.max(np.abs(np.asarray(ref, np.float64) - np.asarray(ref_perturbed, np.float64))))
    ok = (d <= ABS_TOL and r <= REL_TOL) or d <= factor * floor
    assert ok, f"{what}: max|d|={d:.3e} rel={r:.3e}; one-ulp input floor {floor:.3e} (x{factor})"
    return d, floor
