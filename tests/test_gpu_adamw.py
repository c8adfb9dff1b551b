"""GPU AdamW step of the adapters against the fp64 oracle, with the
optimizer state in device memory and in paged (unified) memory moved to the
host and back between steps; argument checks."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

# hyper-parameters as the fp32 values the kernel computes with, so that the
# fp64 oracle starts from the same numbers
HP = {k: float(np.float32(v)) for k, v in
      dict(lr=2e-4, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01, grad_scale=0.5).items()}


def _close(got, ref, scale, what):
    got = np.asarray(got, np.float64)
    err = np.abs(got - ref)
    tol = 4e-6 * (np.abs(ref) + scale)
    assert np.all(err <= tol), f"{what}: max err {err.max():.3e}, worst ratio {(err / tol).max():.2f}"


def _run(Q, O, n, steps, paged):
    rng = np.random.default_rng(n)
    p0 = rng.normal(0, 0.05, n).astype(np.float32)
    grads = [rng.normal(0, 1e-3, n).astype(np.float32) for _ in range(steps)]
    p = torch.from_numpy(p0.copy()).cuda()
    pb = torch.empty(n, dtype=torch.bfloat16, device="cuda")
    if paged:
        m = Q.PagedBuffer(4 * n)
        v = Q.PagedBuffer(4 * n)
        m.host_view(np.float32)[:] = 0
        v.host_view(np.float32)[:] = 0
    else:
        m = torch.zeros(n, device="cuda")
        v = torch.zeros(n, device="cuda")
    rp, rm, rv = p0.astype(np.float64), np.zeros(n), np.zeros(n)
    mag = np.zeros(n)  # size of the terms summed into m (it can cancel to near 0)
    for t, g in enumerate(grads, start=1):
        mag = HP["beta1"] * mag + (1 - HP["beta1"]) * np.abs(g.astype(np.float64)) * HP["grad_scale"]
        if paged:
            # the state starts the step in host memory (paged out); the
            # kernel's accesses bring it back (odd steps: on demand; even
            # steps: an explicit prefetch to the device)
            m.prefetch(to_host=True)
            v.prefetch(to_host=True)
            if t % 2 == 0:
                m.prefetch(to_host=False)
                v.prefetch(to_host=False)
        Q.qlora_adamw_step(p, m, v, torch.from_numpy(g).cuda(), pb, step=t, **HP)
        O.adamw_step(rp, rm, rv, g, step=t, **HP)
    torch.cuda.synchronize()
    assert Q.qlora_get_last_error() == 0
    gm = m.host_view(np.float32).copy() if paged else m.cpu().numpy()
    gv = v.host_view(np.float32).copy() if paged else v.cpu().numpy()
    _close(p.cpu().numpy(), rp, HP["lr"], "param")
    _close(gm, rm, mag, "exp_avg")
    _close(gv, rv, 1e-18, "exp_avg_sq")
    # the bf16 copy is the rounding of the fp32 master
    assert torch.equal(pb.view(torch.int16), p.to(torch.bfloat16).view(torch.int16))
    return p.cpu(), gm, gv


@pytest.mark.parametrize("n", [4, 1003, 1 << 20])
def test_adamw_parity(Q, O, cuda, n):
    _run(Q, O, n, 3, paged=False)


def test_adamw_paged_state_matches_device_state(Q, O, cuda):
    n = 65536 + 5
    a = _run(Q, O, n, 4, paged=True)
    b = _run(Q, O, n, 4, paged=False)
    assert torch.equal(a[0], b[0])
    assert np.array_equal(a[1], b[1]) and np.array_equal(a[2], b[2])


def test_adamw_rejects(Q, cuda):
    p = torch.zeros(16, device="cuda")
    with pytest.raises(Q.QloraError):
        Q.qlora_adamw_step(p, p, p, p, step=0, lr=1e-3)
    with pytest.raises(Q.QloraError):
        Q.qlora_adamw_step(p, p, p, p, step=1, lr=1e-3, beta1=1.0)
    with pytest.raises(Q.QloraError):
        Q.qlora_adamw_step(p[1:], p[1:], p[1:], p[1:], step=1, lr=1e-3)  # not 16-byte aligned
