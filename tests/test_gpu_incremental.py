"""Incremental pooled-key cache on the GPU: dsa_indexer_store and
dsa_kpool_compress_tokens against the oracle and against the full compress.

The caches use the capacity layout an incremental decode needs: request b owns
a fixed block of rows (req_start does not move between steps) and its rows past
the current length are invalid. A step stores its new rows (marked valid) and
recomputes only the pools that hold them; the result must equal, byte for byte,
what the full compress writes for the updated cache.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle as O
from gpu_helpers import assert_keys_close, dev_bits, device_status_clean, host_bits
from sparse_attention_indexer_head_b200 import workloads as W

pytestmark = pytest.mark.gpu

CANARY = 0x7F


@pytest.fixture(scope="module")
def B():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_attention_indexer_head_b200 import build
    build.build()
    from sparse_attention_indexer_head_b200 import binding
    binding.dsa_device_status(reset=True)
    return binding


def _i32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()


def _u8(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint8)).cuda()


class Cache:
    """Device indexer cache (k, gate, valid) plus the layer's compress weights."""

    def __init__(self, wl):
        self.wl = wl
        self.k = dev_bits(wl.k)
        self.gate = dev_bits(wl.gate)
        self.valid = _u8(wl.valid)
        self.req_start = _i32(wl.req_start)
        self.ape = torch.from_numpy(wl.ape).cuda()
        self.ln_w = dev_bits(wl.ln_w)
        self.ln_b = dev_bits(wl.ln_b)

    def outputs(self):
        wl = self.wl
        t = dict(keys=torch.empty(wl.B, wl.max_pools, 128, dtype=torch.bfloat16, device="cuda"),
                 idx=torch.empty(wl.B, wl.max_pools, wl.kpool, dtype=torch.int32, device="cuda"),
                 pv=torch.empty(wl.B, wl.max_pools, dtype=torch.uint8, device="cuda"),
                 fv=torch.empty(wl.B, dtype=torch.int32, device="cuda"))
        for x in t.values():
            x.view(torch.uint8).fill_(CANARY)
        return t

    def compress(self, B, o):
        wl = self.wl
        B.dsa_kpool_compress(self.k, self.gate, self.valid, self.req_start, wl.B, 128, wl.kpool,
                             wl.max_pools, self.ape, self.ln_w, self.ln_b, wl.eps, o["keys"],
                             o["idx"], o["pv"], o["fv"])

    def compress_tokens(self, B, o, begin, end):
        wl = self.wl
        B.dsa_kpool_compress_tokens(self.k, self.gate, self.valid, self.req_start, wl.B, 128,
                                    wl.kpool, wl.max_pools, self.ape, self.ln_w, self.ln_b, wl.eps,
                                    _i32(begin), _i32(end), o["keys"], o["idx"], o["pv"], o["fv"])

    def store(self, B, k_new, g_new, v_new, tok_req, tok_pos):
        wl = self.wl
        B.dsa_indexer_store(dev_bits(k_new), dev_bits(g_new),
                            None if v_new is None else _u8(v_new), _i32(tok_req), _i32(tok_pos),
                            len(tok_req), 128, self.req_start, wl.B, self.k, self.gate, self.valid)

    def host(self):
        return host_bits(self.k), host_bits(self.gate), self.valid.cpu().numpy()


def _np(o):
    return (host_bits(o["keys"]), o["idx"].cpu().numpy(), o["pv"].cpu().numpy(),
            o["fv"].cpu().numpy())


def _capacity_workload(kpool, caps, lengths, pads, seed=5):
    """Requests with capacity caps[b]; rows < pads[b] and rows >= lengths[b] invalid."""
    mp = max(1, max((c + kpool - 1) // kpool for c in caps))
    wl = W.build(f"capacity k{kpool}", lengths=caps, pads=[0] * len(caps), kpool=kpool,
                 max_pools=mp, select_k=8, hm=16, q_req=[0], q_pos=[0], seed=seed)
    for b, (L, p) in enumerate(zip(lengths, pads)):
        r0 = wl.req_start[b]
        wl.valid[r0:r0 + caps[b]] = 0
        wl.valid[r0 + min(p, L):r0 + L] = 1
    return wl


def _assert_same(a, b, what):
    for x, y, name in zip(a, b, ("pool_keys", "pool_idx", "pool_valid", "first_valid")):
        assert np.array_equal(x, y), f"{what}: {name} differs"


def test_indexer_store_bit_exact(B):
    wl = _capacity_workload(4, [40, 0, 77, 9], [10, 0, 77, 3], [0, 0, 5, 0])
    c = Cache(wl)
    rng = np.random.default_rng(7)
    n = 37
    k_new = W.f32_to_bf16_bits(rng.standard_normal((n, 128), dtype=np.float32))
    g_new = W.f32_to_bf16_bits(rng.standard_normal((n, 128), dtype=np.float32))
    v_new = rng.integers(0, 3, n).astype(np.uint8)            # 0, 1 and 2 (nonzero -> 1)
    tok_req = rng.integers(-1, 5, n).astype(np.int32)         # -1 and 4 are no request
    tok_pos = rng.integers(-2, 80, n).astype(np.int32)
    # distinct destination rows (two rows for one slot would race)
    seen, keep = set(), []
    for i in range(n):
        key = (int(tok_req[i]), int(tok_pos[i]))
        if key not in seen:
            seen.add(key)
            keep.append(i)
    keep = np.asarray(keep)
    k_new, g_new, v_new, tok_req, tok_pos = (a[keep] for a in (k_new, g_new, v_new, tok_req, tok_pos))
    want = O.indexer_store(wl.k, wl.gate, wl.valid, wl.req_start, k_new, g_new, v_new, tok_req,
                           tok_pos)
    c.store(B, k_new, g_new, v_new, tok_req, tok_pos)
    torch.cuda.synchronize()
    got = c.host()
    for x, y, name in zip(got, want, ("k", "gate", "valid")):
        np.testing.assert_array_equal(x, y, err_msg=name)
    # valid_new NULL marks every stored token valid
    c2 = Cache(wl)
    c2.store(B, k_new[:5], g_new[:5], None, np.zeros(5, np.int32), np.arange(5, dtype=np.int32))
    torch.cuda.synchronize()
    v = c2.valid.cpu().numpy()
    assert v[:5].all() and np.array_equal(v[5:], wl.valid[5:])
    device_status_clean(B)


@pytest.mark.parametrize("kpool", [1, 2, 3, 4, 5, 6, 7, 8])
def test_compress_tokens_after_append_equals_full_compress(B, kpool):
    #            cap   len  pad   appended
    spec = [(300, 121, 0, 1),        # one decode token, mid-pool
            (300, 128, 7, 3),        # crosses a pool boundary, left padding
            (64, 0, 0, 5),           # empty request gets its first tokens: pool grid moves
            (64, 40, 40, 2),         # all padding so far: first valid token is new
            (129, 129, 0, 0),        # full, nothing appended
            (520, 200, 3, kpool + 2),
            (8, 7, 0, 1)]            # fills the request's last row
    caps = [s[0] for s in spec]
    lens = [s[1] for s in spec]
    pads = [s[2] for s in spec]
    wl = _capacity_workload(kpool, caps, lens, pads, seed=20 + kpool)
    c = Cache(wl)
    inc = c.outputs()
    c.compress(B, inc)                                       # state before the step

    rng = np.random.default_rng(kpool)
    tok_req, tok_pos = [], []
    for b, (cap, L, _, n) in enumerate(spec):
        for j in range(n):
            if L + j < cap:
                tok_req.append(b)
                tok_pos.append(L + j)
    n = len(tok_req)
    k_new = W.f32_to_bf16_bits(rng.standard_normal((n, 128), dtype=np.float32))
    g_new = W.f32_to_bf16_bits(rng.standard_normal((n, 128), dtype=np.float32))
    c.store(B, k_new, g_new, None, tok_req, tok_pos)
    begin = np.array([s[1] for s in spec], np.int32)
    end = np.array([min(s[1] + s[3], s[0]) for s in spec], np.int32)
    c.compress_tokens(B, inc, begin, end)

    full = c.outputs()
    c.compress(B, full)                                      # the updated cache from scratch
    torch.cuda.synchronize()
    got, ref_full = _np(inc), _np(full)
    _assert_same(got, ref_full, f"kpool {kpool}")

    # and against the oracle on the host copy of the updated cache
    hk, hg, hv = c.host()
    exp_k, exp_g, exp_v = O.indexer_store(wl.k, wl.gate, wl.valid, wl.req_start, k_new, g_new,
                                          None, tok_req, tok_pos)
    np.testing.assert_array_equal(hk, exp_k)
    np.testing.assert_array_equal(hv, exp_v)
    keys, idx, pv, fv = O.kpool_compress(exp_k, exp_g, exp_v, wl.req_start, kpool, wl.max_pools,
                                         wl.ape, wl.ln_w, wl.ln_b, wl.eps)
    np.testing.assert_array_equal(got[3], fv)
    np.testing.assert_array_equal(got[2], pv)
    np.testing.assert_array_equal(got[1], idx)
    wl2 = dataclasses.replace(wl, k=exp_k, gate=exp_g, valid=exp_v)
    assert_keys_close(got[0], keys, pv, wl2, fv)
    assert fv[2] == 0 and fv[3] == 40                       # the two requests whose f moved
    device_status_clean(B)


def test_compress_tokens_leaves_other_pools_untouched(B):
    """Pools outside the ranges keep whatever the buffers held (here a canary)."""
    wl = _capacity_workload(4, [256, 256], [100, 100], [0, 0])
    c = Cache(wl)
    o = c.outputs()
    c.compress(B, o)
    torch.cuda.synchronize()
    fv = o["fv"].clone()
    for x in (o["keys"], o["idx"], o["pv"]):
        x.view(torch.uint8).fill_(CANARY)
    o["fv"].copy_(fv)
    c.compress_tokens(B, o, np.array([97, 0]), np.array([99, 0]))   # request 1: empty range
    torch.cuda.synchronize()
    keys, idx, pv, _ = _np(o)
    touched = np.zeros((2, wl.max_pools), bool)
    touched[0, 24] = True                                            # tokens 97, 98 -> pool 24
    canary16 = np.uint16(CANARY | (CANARY << 8))
    assert (keys[~touched] == canary16).all()
    assert (pv[~touched] == CANARY).all()
    assert (idx[~touched] == np.int32(0x7F7F7F7F)).all()
    assert pv[0, 24] == 1 and (idx[0, 24] == np.arange(96, 100)).all()
    full = c.outputs()
    c.compress(B, full)
    torch.cuda.synchronize()
    kf, _, _, _ = _np(full)
    assert np.array_equal(keys[0, 24], kf[0, 24])
    device_status_clean(B)


def test_compress_tokens_first_valid_unknown_recomputes_all(B):
    """first_valid = -1 on entry: every pool of the request is written, equal to full."""
    wl = _capacity_workload(3, [100, 50, 0], [100, 20, 0], [9, 0, 0])
    c = Cache(wl)
    o = c.outputs()
    o["fv"].fill_(-1)
    c.compress_tokens(B, o, np.zeros(3, np.int32), np.zeros(3, np.int32))   # empty ranges
    full = c.outputs()
    c.compress(B, full)
    torch.cuda.synchronize()
    _assert_same(_np(o), _np(full), "first_valid -1")
    device_status_clean(B)


@pytest.mark.parametrize("name", ["tiny", "batched"])
def test_incremental_step_equals_full_step(B, name):
    """A decode step through store + token-range compress gives the full step's outputs."""
    from sparse_attention_indexer_head_b200.pipeline import DecodeStep
    wl = W.make(name)
    full = DecodeStep(wl)
    full.run()
    inc = DecodeStep(wl)
    inc.kpool_compress()                     # the cache's pooled keys before the step
    inc.stage_new_tokens()
    for _ in range(2):                       # repeated steps stay consistent
        inc.run_incremental()
    torch.cuda.synchronize()
    a, b = full.outputs_numpy(), inc.outputs_numpy()
    for key in a:
        assert np.array_equal(a[key], b[key], equal_nan=key in ("scores", "lse")), key
    device_status_clean(B)


@pytest.mark.parametrize("kpool", [3, 4])
def test_decode_sequence_stays_equal_to_full_compress(B, kpool):
    """Twelve decode steps, each storing one new token per request (some invalid,
    some requests idle), through one captured CUDA graph: after every step the
    incremental outputs equal the full compress of the grown cache, byte for byte."""
    caps = [96, 64, 80, 33]
    lens = [40, 0, 77, 10]                  # request 1 starts empty
    wl = _capacity_workload(kpool, caps, lens, [3, 0, 0, 0], seed=60 + kpool)
    c = Cache(wl)
    inc = c.outputs()
    c.compress(B, inc)
    rng = np.random.default_rng(kpool + 100)
    nb = wl.B
    # device-side step inputs, refilled in place each step so a graph can replay them
    k_new = torch.empty(nb, 128, dtype=torch.bfloat16, device="cuda")
    g_new = torch.empty_like(k_new)
    v_new = torch.empty(nb, dtype=torch.uint8, device="cuda")
    t_req = torch.arange(nb, dtype=torch.int32, device="cuda")
    t_pos = torch.empty(nb, dtype=torch.int32, device="cuda")
    t_beg = torch.empty(nb, dtype=torch.int32, device="cuda")
    t_end = torch.empty(nb, dtype=torch.int32, device="cuda")

    def step(stream=None):
        B.dsa_indexer_store(k_new, g_new, v_new, t_req, t_pos, nb, 128, c.req_start, nb, c.k,
                            c.gate, c.valid, stream)
        B.dsa_kpool_compress_tokens(c.k, c.gate, c.valid, c.req_start, nb, 128, kpool,
                                    wl.max_pools, c.ape, c.ln_w, c.ln_b, wl.eps, t_beg, t_end,
                                    inc["keys"], inc["idx"], inc["pv"], inc["fv"], stream)

    s = torch.cuda.Stream()
    graph = torch.cuda.CUDAGraph()
    pos = np.array(lens)

    def fill():
        active = (rng.random(nb) < 0.8) & (pos < np.array(caps))
        k_new.copy_(dev_bits(W.f32_to_bf16_bits(rng.standard_normal((nb, 128), dtype=np.float32))))
        g_new.copy_(dev_bits(W.f32_to_bf16_bits(rng.standard_normal((nb, 128), dtype=np.float32))))
        v_new.copy_(_u8((rng.random(nb) < 0.9).astype(np.uint8)))
        p = np.where(active, pos, -1).astype(np.int32)        # -1: no new token this step
        t_pos.copy_(_i32(p))
        t_beg.copy_(_i32(np.where(active, pos, 0)))
        t_end.copy_(_i32(np.where(active, pos + 1, 0)))
        return active

    for it in range(12):
        active = fill()
        torch.cuda.synchronize()
        if it == 0:
            with torch.cuda.stream(s):
                step()                                        # eager first (sets attributes)
            s.synchronize()
            with torch.cuda.graph(graph, stream=s):
                step()
        else:
            graph.replay()
        torch.cuda.synchronize()
        pos = pos + active
        full = c.outputs()
        # the full reference must start from the same unwritten-row contents
        full["keys"].copy_(inc["keys"])
        c.compress(B, full)
        torch.cuda.synchronize()
        _assert_same(_np(inc), _np(full), f"step {it}")
    del graph
    device_status_clean(B)


def test_streamed_decode_matches_eager_steps(B):
    """StreamedDecode (H2D, the step and D2H in one graph per slot, consecutive steps on
    two streams) returns each step's output exactly as an eager step on the same
    inputs does."""
    from sparse_attention_indexer_head_b200.pipeline import (QUERY_INPUTS, DecodeStep,
                                                            StreamedDecode, host_tensors)
    wl_a, wl_b = W.make("tiny", seed=0), W.make("tiny", seed=1)
    ins = [{k: host_tensors(w)[k].pin_memory() for k in QUERY_INPUTS} for w in (wl_a, wl_b)]
    ref = []
    for q in ins:
        st = DecodeStep(wl_a)
        for k, v in q.items():
            st.t[k].copy_(v)
        st.run()
        torch.cuda.synchronize()
        ref.append(st.out.view(torch.int16).cpu().numpy())
    sd = StreamedDecode(wl_a, slots=2)
    got = []
    for i in range(7):
        sd.write_inputs(i, ins[i % 2])       # its slot's previous step was read (below)
        sd.submit()
        if i >= 1:
            got.append(sd.result(i - 1).view(torch.int16).numpy().copy())
    got.append(sd.result(6).view(torch.int16).numpy().copy())
    for i, g in enumerate(got):
        assert np.array_equal(g, ref[i % 2]), i
    assert not np.array_equal(ref[0], ref[1])
    device_status_clean(B)
