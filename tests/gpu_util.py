"""Helpers for the GPU parity tests (tolerances follow the acceptance bar:
rel-L2 <= 1e-5 for fp32 outputs, <= 1e-2 for bf16 outputs, max logit within
1e-3 relative per head, clipped-head sets and clipped weights bit-exact)."""
import numpy as np

TOL_F32 = 1e-5
TOL_BF16 = 1e-2
TOL_MAXLOGIT = 1e-3


def rel_l2(got, want) -> float:
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    return float(np.linalg.norm(got - want) / np.linalg.norm(want))


def max_rel(got, want) -> float:
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    return float(np.max(np.abs(got - want) / np.abs(want)))


def per_head(fn, heads, workers=8):
    """Run the oracle one head at a time on a thread pool: fn(h) -> that head's
    result.  numpy releases the GIL in its matrix products and elementwise
    passes, so the heads of a long sequence overlap; each head's arithmetic is
    the oracle's own, unchanged."""
    from concurrent.futures import ThreadPoolExecutor
    heads = list(heads)
    with ThreadPoolExecutor(max(1, min(workers, len(heads)))) as ex:
        return dict(zip(heads, ex.map(fn, heads)))


def dev(a, dtype, device="cuda"):
    from gated_mla_qk_b200 import synth
    return None if a is None else synth.to_torch(a, dtype, device)


def host(t) -> np.ndarray:
    import torch
    return t.detach().to("cpu", torch.float32).numpy() if t.dtype != torch.uint8 else t.cpu().numpy()


def check_status():
    import gated_mla_qk_b200 as gm
    st = gm.device_status()
    assert st == 0, f"device status {st}"


PAD = 4096          # guard bytes on each side; keeps the 16-byte (and 512-byte) alignment of the output


class Guarded:
    """A [PAD | nbytes | PAD] device buffer whose middle is viewed as ``shape`` of ``dtype``."""

    def __init__(self, shape, dtype, init=None):
        import torch
        self.shape, self.dtype = tuple(shape), dtype
        self.nbytes = int(np.prod(self.shape)) * torch.empty(0, dtype=dtype).element_size()
        self.buf = torch.full((PAD + self.nbytes + PAD,), 0xFF, dtype=torch.uint8, device="cuda")
        self.t = self.buf[PAD:PAD + self.nbytes].view(dtype).view(self.shape)
        if init is not None:
            self.t.copy_(init)

    def check(self, name, written=True):
        import torch
        lo, hi = self.buf[:PAD], self.buf[PAD + self.nbytes:]
        assert bool((lo == 0xFF).all()), f"{name}: bytes before the output were written"
        assert bool((hi == 0xFF).all()), f"{name}: bytes after the output were written"
        if written and self.dtype in (torch.float32, torch.bfloat16):
            assert not bool(torch.isnan(self.t).any()), f"{name}: part of the output was never written"


def guarded_bytes(n):
    import torch
    return Guarded((n,), torch.uint8)
