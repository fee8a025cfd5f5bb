"""GPU parity on seeded random shapes: the whole call (profiling, layout
transformation, block-sparse attention, inverse layout) against the fp64
oracle, over ragged and degenerate sizes the fixed cases do not reach.

Each case draws B, H, N frames, F positions (L = N F up to 3000, F = 1 and
N = 1 included), d, the band half-widths a1 in [1, N + 1] and a2 in
[1, F + 2] (bands wider than the video included), the sampled row count S, the
tensor layout and the input type.  Checks, as in test_gpu_parity:
  * MSEs within the rounding bound of the oracle's, labels equal wherever the
    oracle's gap decides them;
  * the output against the oracle's sparse attention under the call's own
    labels: bf16 max-abs 2e-2 / relative L2 1e-2, fp32 1e-4 / 1e-5, tf32
    1e-2 / 4e-3 (the bars of test_gpu_tf32);
  * the device status word stays clear.
"""
import numpy as np
import pytest
import torch

import oracle
from sparse_attention_video_profile_b200 import svg
from test_gpu_parity import DEV, check_profile, f64, profile_bounds

TOLS = {"bf16": (2e-2, 1e-2), "fp32": (1e-4, 1e-5), "tf32": (1e-2, 4e-3)}
N_CASES = 40


def draw_case(i):
    rng = np.random.default_rng(1000 + i)
    kind = ["bf16", "bf16", "bf16", "fp32", "tf32"][i % 5]
    while True:
        N = int(rng.integers(1, 13))
        F = int(rng.choice([1, 2, 7, 37, 64, 128, 129, 250, 300, 400]))
        if N * F <= 3000:
            break
    d = int(rng.choice([64, 128])) if kind == "bf16" else int(rng.choice([32, 64, 128]))
    L = N * F
    return dict(kind=kind, B=int(rng.integers(1, 3)), H=int(rng.integers(1, 4)), N=N, F=F, d=d,
                a1=int(rng.integers(1, N + 2)), a2=int(rng.integers(1, F + 3)),
                S=int(rng.integers(1, min(L, 128) + 1)), layout=str(rng.choice(["bhld", "blhd"])),
                seed=int(rng.integers(0, 2 ** 31)))


CASES = [draw_case(i) for i in range(N_CASES)]


def _id(c):
    return "{kind}-B{B}H{H}N{N}F{F}d{d}-a{a1},{a2}-S{S}-{layout}".format(**c)


@pytest.mark.gpu
@pytest.mark.parametrize("case", CASES, ids=_id)
def test_whole_call_random_shapes(case):
    c = case
    B, H, N, F, d = c["B"], c["H"], c["N"], c["F"], c["d"]
    L = N * F
    g = torch.Generator(device=DEV)
    g.manual_seed(c["seed"])
    dtype = torch.bfloat16 if c["kind"] == "bf16" else torch.float32
    # [B, H, L, d] values; the call sees them in the drawn layout
    qkv = [(torch.randn(B, H, L, d, generator=g, device=DEV) * 0.7).to(dtype) for _ in range(3)]
    blhd = c["layout"] == "blhd"
    args = [t.transpose(1, 2).contiguous() if blhd else t for t in qkv]
    rows_np = np.sort(np.random.default_rng(c["seed"]).choice(L, c["S"], replace=False)).astype(np.int32)
    rows = torch.from_numpy(rows_np).to(DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o, mse, label = svg.svg_sparse_3d_attn(*args, N, F, c["a1"], c["a2"], rows, status=status,
                                           layout=c["layout"], tf32=c["kind"] == "tf32")
    torch.cuda.synchronize()
    assert int(status.item()) == 0, f"device status {int(status.item())}"
    if blhd:
        o = o.transpose(1, 2)
    qn, kn, vn = (f64(t) for t in qkv)
    ref_mse, ref_label = oracle.profile_heads(qn, kn, vn, N, F, c["a1"], c["a2"], rows_np)
    check_profile(mse, label, ref_mse, ref_label,
                  profile_bounds(qn, kn, vn, N, F, c["a1"], c["a2"], rows_np, fp32=dtype == torch.float32))
    ref = oracle.sparse_attention(qn, kn, vn, label.cpu().numpy(), N, F, c["a1"], c["a2"])
    got = f64(o)
    assert np.all(np.isfinite(got))
    max_abs = float(np.max(np.abs(got - ref)))
    rel = float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30))
    ta, tr = TOLS[c["kind"]]
    assert max_abs <= ta and rel <= tr, f"max_abs {max_abs:.3e} rel_l2 {rel:.3e}"


def test_cases_cover_the_edges():
    """The drawn cases reach the degenerate sizes and bands they are meant to."""
    assert any(c["F"] == 1 for c in CASES) or any(c["N"] == 1 for c in CASES)
    assert any(c["a1"] > c["N"] for c in CASES) and any(c["a2"] > c["F"] for c in CASES)
    assert {c["layout"] for c in CASES} == {"bhld", "blhd"}
    assert {c["kind"] for c in CASES} == {"bf16", "fp32", "tf32"}
    assert any(c["N"] * c["F"] % 128 for c in CASES)
