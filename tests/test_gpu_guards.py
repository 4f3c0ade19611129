"""Out-of-bounds writes, found without a sanitizer: every buffer a step touches is allocated with
guard regions before and after it, filled with a sentinel pattern, and after several steps
(ragged sizes, odd Nd, a ragged bucket or layer, an overflowing step, aligned and unaligned
starts) every guard must still hold the sentinel.  Covers each path of zero_step."""
import numpy as np
import pytest
import torch

import synth
import zero_sharded_optimizer_03_b200 as zero

pytestmark = pytest.mark.gpu

G = 64  # guard elements on each side: keeps 16-byte alignment for 1-, 2- and 4-byte elements
SENTINEL = {1: 0x5A, 2: 0x7E57, 4: 0x7E577E57}
VIEW = {1: torch.uint8, 2: torch.int16, 4: torch.int32}


class Guarded:
    """A device buffer of n elements with G sentinel elements on each side; `shift` extra
    elements before the body make its start unaligned."""

    def __init__(self, n, dtype, shift=0):
        self.n = max(n, 1)
        self.t = torch.empty(self.n + 2 * G + shift, dtype=dtype, device="cuda")
        self.size = self.t.element_size()
        self.t.view(VIEW[self.size]).fill_(SENTINEL[self.size])
        self.lo = G + shift
        self.body = self.t[self.lo:self.lo + self.n]
        self.body.zero_()

    def ptr(self):
        return self.body.data_ptr()

    def intact(self):
        v = self.t.view(VIEW[self.size])
        s = SENTINEL[self.size]
        return bool((v[:self.lo] == s).all()) and bool((v[self.lo + self.n:] == s).all())


def _stream():
    return torch.cuda.current_stream().cuda_stream


PATHS = [("fused", 2, zero.ZERO_FUSED, 0), ("fused-unaligned", 2, zero.ZERO_FUSED, 1),
         ("tma", 2, zero.ZERO_FUSED | zero.ZERO_FORCE_TMA, 0),
         ("two-pass", 2, zero.ZERO_TWO_PASS, 0), ("two-pass-unaligned", 2, zero.ZERO_TWO_PASS, 1),
         ("zero3", 3, zero.ZERO_FUSED, 0), ("zero3-unaligned", 3, zero.ZERO_FUSED, 1),
         ("zero3-tma-gather", 3, zero.ZERO_FORCE_TMA, 0),
         ("zero3-fused-layers", 3, zero.ZERO_FUSED_LAYERS, 0)]


@pytest.mark.parametrize("name,stage,flags,shift", PATHS, ids=[p[0] for p in PATHS])
def test_steps_write_nothing_outside_their_buffers(name, stage, flags, shift):
    Nd, N = 3, 2048 * 5 + 13
    L = 4096  # stage 3: layers of 4096, 4096 and 2061 elements
    bucket = 3001 if stage != 3 else L
    if stage == 3:
        sizes = [min(L, N - k) for k in range(0, N, L)]
        Np = sum(zero.zero_partition(x, Nd).Np for x in sizes)
    else:
        Np = zero.zero_partition(N, Nd).Np
    bufs = []

    def buf(n, dtype):
        b = Guarded(n, dtype, shift)
        bufs.append(b)
        return b

    grads = [buf(N, torch.bfloat16) for _ in range(Nd)]
    params = [buf(N, torch.bfloat16) for _ in range(Nd)]
    two_copies = (stage != 3 and not flags & zero.ZERO_TWO_PASS) or flags & zero.ZERO_FUSED_LAYERS
    copies = 2 if two_copies else 1
    master = [buf(Np, torch.float32) for _ in range(copies)]
    exp_avg = [buf(Np, torch.float32) for _ in range(copies)]
    exp_avg_sq = [buf(Np, torch.float32) for _ in range(copies)]
    need_gshard = flags & zero.ZERO_TWO_PASS or (stage == 3 and not flags & zero.ZERO_FUSED_LAYERS)
    gshard = buf(Np, torch.float32) if need_gshard else None
    pshard = buf(Np, torch.bfloat16) if stage == 3 else None
    ws = Guarded(zero.zero_workspace_bytes(), torch.uint8)  # the workspace itself stays aligned
    bufs.append(ws)

    st = zero.zero_state_t()
    st.grad_dtype = zero.ZERO_BF16
    st.flags = flags
    for r in range(Nd):
        st.grads[r] = grads[r].ptr()
        st.params[r] = params[r].ptr()
    for k in range(copies):
        st.master[k] = master[k].ptr()
        st.exp_avg[k] = exp_avg[k].ptr()
        st.exp_avg_sq[k] = exp_avg_sq[k].ptr()
    if gshard is not None:
        st.grad_shard = gshard.ptr()
    if pshard is not None:
        st.param_shard = pshard.ptr()
    if stage == 3:
        st.grad_layer_stride = L
        st.param_layer_stride = L
    st.workspace = ws.ptr()

    # initial weights in the real elements (padding stays zero), bf16 copies where the step reads them
    synth.fill_device(master[0].ptr(), synth.NORMAL, synth.F32, synth.SEED, synth.MASTER_STREAM,
                      Np, 0.02, cuda_stream=_stream())
    if stage == 3:
        off = 0
        for x in sizes:
            p = zero.zero_partition(x, Nd).Np
            master[0].body[off + x:off + p].zero_()
            off += p
        zero.zero_allgather(master[0].ptr(), [pshard.ptr()], 1, 0, Np, zero.ZERO_GATE_ALWAYS, None,
                            _stream())
    else:
        master[0].body[N:].zero_()
        zero.zero_allgather(master[0].ptr(), [p.ptr() for p in params], Nd, 0, N,
                            zero.ZERO_GATE_ALWAYS, None, _stream())
    zero.zero_workspace_init(ws.ptr(), 0, _stream())
    hp = zero.hparams(lr=1e-3, weight_decay=0.01)
    for k in (1, 2, 3):
        for r in range(Nd):
            synth.fill_device(grads[r].ptr(), synth.NORMAL, synth.BF16, synth.SEED,
                              synth.grad_stream(k, r), N, 1e-3, cuda_stream=_stream())
        if k == 2:  # an overflowing step: the skip and repair paths run too
            grads[1].body.view(torch.int16)[N // 2] = int(np.array([0x7F80], np.uint16).view(np.int16)[0])
        zero.zero_step(stage, Nd, N, bucket, st, hp, _stream())
    torch.cuda.synchronize()
    res = zero.zero_read_result(ws.ptr(), _stream())
    assert (res["step"], res["skipped"], res["error"]) == (2, 1, 0), res
    broken = [i for i, b in enumerate(bufs) if not b.intact()]
    assert not broken, "%s: writes outside buffers %s" % (name, broken)
