"""Comparison helpers for the GPU-vs-oracle parity tests (tolerances from the method's acceptance
criteria: selection bit-exact except near-ties with cutoff margin < 1e-4; attention output max abs
error <= 1e-2 and mean abs error <= 1e-3; L_KL relative error <= 1e-4; gradients max abs error
<= 1e-3)."""
import numpy as np

NEAR_TIE = 1e-4
ATT_MAX, ATT_MEAN = 1e-2, 1e-3
LSE_MAX = 2e-3
KL_REL = 1e-4
GRAD_MAX = 1e-3
GRAD_REL = 2e-3  # stricter check used alongside: max error relative to the largest gradient entry


# Near-tie rows excluded by each selection comparison of the session, as (test id, (row, group)
# pairs compared, near-tie pairs, near-tie pairs whose selection differs); printed at the end of the
# run by the terminal summary in conftest.py.
CURRENT_TEST = ""
NEAR_TIE_LOG = []
# Achieved errors that a test chooses to report (printed with the near-tie summary).
REPORT_LOG = []


def report(line: str) -> None:
    REPORT_LOG.append((CURRENT_TEST, line))


def compare_blocks(gpu_blocks, ora_blocks, margin):
    """Bit-exact equality of the selected block ids for every (row, group) whose cutoff margin is
    >= NEAR_TIE; returns (number of mismatching rows outside near-ties, number of near-tie rows).
    The near-tie count of every comparison is logged for the session report."""
    g = np.asarray(gpu_blocks).reshape(-1, gpu_blocks.shape[-1])
    o = np.asarray(ora_blocks).reshape(-1, ora_blocks.shape[-1])
    m = np.asarray(margin).reshape(-1)
    near = m < NEAR_TIE
    differ = np.any(g != o, axis=1)
    bad = differ & ~near
    NEAR_TIE_LOG.append((CURRENT_TEST, int(g.shape[0]), int(near.sum()), int((differ & near).sum())))
    return int(bad.sum()), int(near.sum())


def check_attention(out_gpu, out_ref, lse_gpu=None, lse_ref=None):
    e = np.abs(np.asarray(out_gpu, dtype=np.float64) - np.asarray(out_ref, dtype=np.float64))
    assert e.max() <= ATT_MAX, f"attention max abs error {e.max():.3e}"
    assert e.mean() <= ATT_MEAN, f"attention mean abs error {e.mean():.3e}"
    if lse_gpu is not None:
        le = np.abs(np.asarray(lse_gpu, dtype=np.float64) - np.asarray(lse_ref, dtype=np.float64))
        assert le.max() <= LSE_MAX, f"lse max abs error {le.max():.3e}"
    return float(e.max()), float(e.mean())


def check_attention_bf16(out_gpu, out_ref):
    """A bf16-stored output: the fp32 bound plus the storage rounding, half a bf16 unit in the last
    place (bf16 keeps 8 significant bits, so at most 2^-8 |o|)."""
    g = np.asarray(out_gpu, dtype=np.float64)
    r = np.asarray(out_ref, dtype=np.float64)
    e = np.abs(g - r)
    bound = ATT_MAX + 2.0 ** -8 * np.abs(r)
    assert (e <= bound).all(), f"bf16 attention error {e.max():.3e} above its bound"
    assert e.mean() <= ATT_MEAN + 2.0 ** -8 * np.abs(r).mean(), f"bf16 attention mean abs error {e.mean():.3e}"
    return float(e.max())


def check_grad(g_gpu, g_ref, name):
    g = np.asarray(g_gpu, dtype=np.float64)
    r = np.asarray(g_ref, dtype=np.float64)
    e = np.abs(g - r).max()
    scale = max(np.abs(r).max(), 1e-30)
    assert e <= GRAD_MAX, f"{name} max abs error {e:.3e}"
    assert e <= GRAD_REL * scale, f"{name} max error {e:.3e} vs largest entry {scale:.3e}"
    return float(e), float(e / scale)


# Attention backward (derivation in the design notes): P and dS enter the tensor cores as bf16
# (relative rounding 2^-9), and the forward's O and LSE used for g.o and P carry ~1e-3 relative
# error. The gradients are sums over |J| terms with cancellation (the logit gradients of a row sum
# to zero), so errors are measured against the largest entry of each tensor. A tensor that is zero
# in exact arithmetic (a single token attending to itself has dS = 0) keeps fp32 rounding noise:
# the largest entry is floored at BWD_FLOOR for the comparison.
BWD_MAX_REL = 1e-2
BWD_MEAN_REL = 1e-3
BWD_FLOOR = 1e-2


def check_bwd(g_gpu, g_ref, name):
    g = np.asarray(g_gpu, dtype=np.float64)
    r = np.asarray(g_ref, dtype=np.float64)
    scale = max(np.abs(r).max(), BWD_FLOOR)
    e = np.abs(g - r)
    assert e.max() <= BWD_MAX_REL * scale, f"{name}: max error {e.max():.3e} vs largest entry {scale:.3e}"
    assert e.mean() <= BWD_MEAN_REL * scale, f"{name}: mean error {e.mean():.3e} vs largest entry {scale:.3e}"
    return float(e.max() / scale), float(e.mean() / scale)
