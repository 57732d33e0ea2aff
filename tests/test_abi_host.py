"""The C-ABI library on the host (no GPU): it loads, exports every symbol the
header declares, and refuses bad arguments with the documented status before
launching anything."""
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dsa.h")


@pytest.fixture(scope="module")
def B():
    from sparse_attention_indexer_head_b200 import build
    build.build()
    from sparse_attention_indexer_head_b200 import binding
    return binding


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dsa_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_five_stages():
    names = declared_functions()
    for n in ("dsa_head_gate", "dsa_kpool_compress", "dsa_index_scores", "dsa_topk_expand",
              "dsa_sparse_mla_decode"):
        assert n in names


def test_every_declared_symbol_is_exported(B):
    for name in declared_functions():
        assert hasattr(B.lib, name), name
    assert set(declared_functions()) == set(B.EXPORTS)


def test_status_strings_and_version(B):
    assert B.dsa_abi_version() == 1
    for code, name in [(0, "DSA_OK"), (1, "DSA_ERR_INVALID_ARG"), (2, "DSA_ERR_UNSUPPORTED"),
                       (3, "DSA_ERR_ALIGNMENT"), (4, "DSA_ERR_WORKSPACE"), (5, "DSA_ERR_CUDA")]:
        assert B.dsa_status_string(code) == name
    assert B.dsa_status_string(99) == "DSA_ERR_UNKNOWN"


FAKE = 1 << 20          # a 16-byte aligned non-null address; never dereferenced on these paths


def test_selftest_refusals(B):
    assert B.lib.dsa_selftest_bounded_wait(None, None) == B.DSA_ERR_INVALID_ARG
    assert B.lib.dsa_selftest_bounded_wait(FAKE + 2, None) == B.DSA_ERR_ALIGNMENT


def test_head_gate_refusals(B):
    L = B.lib
    assert L.dsa_head_gate(None, None, None, 4, 4096, 16, None) == B.DSA_ERR_INVALID_ARG
    assert L.dsa_head_gate(FAKE, FAKE, FAKE, 4, 4096, 17, None) == B.DSA_ERR_UNSUPPORTED
    assert L.dsa_head_gate(FAKE, FAKE, FAKE, 4, 4094, 16, None) == B.DSA_ERR_UNSUPPORTED
    assert L.dsa_head_gate(FAKE + 4, FAKE, FAKE, 4, 4096, 16, None) == B.DSA_ERR_ALIGNMENT
    assert L.dsa_head_gate(FAKE, FAKE, FAKE, -1, 4096, 16, None) == B.DSA_ERR_INVALID_ARG
    assert L.dsa_head_gate(None, None, None, 0, 4096, 16, None) == B.DSA_OK   # M == 0: no-op


def test_head_gate_routing_predicate(B):
    assert B.dsa_head_gate_supported(16, 4096, 16)
    assert B.dsa_head_gate_supported(0, 4096, 16)                 # empty batch: served (no-op)
    assert not B.dsa_head_gate_supported(16, 4096, 17)            # more than 16 heads
    assert not B.dsa_head_gate_supported(16, 4094, 16)            # K not a multiple of 4
    assert B.lib.dsa_head_gate_supported(-1, 4096, 16) == B.DSA_ERR_INVALID_ARG
    # the predicate and the call agree on every shape
    for M, K, N in [(16, 4096, 16), (3, 4, 1), (5, 4096, 17), (2, 4098, 8), (-1, 8, 1)]:
        want = B.lib.dsa_head_gate_supported(M, K, N)
        got = B.lib.dsa_head_gate(FAKE, FAKE, FAKE, M, K, N, None) if want != B.DSA_OK else want
        assert got == want


def _compress(lib, **kw):
    a = dict(k=FAKE, gate=FAKE, valid=FAKE, req_start=FAKE, B=2, D=128, kpool=4, max_pools=8,
             ape=FAKE, ln_w=FAKE, ln_b=FAKE, eps=1e-5, keys=FAKE, idx=FAKE, pv=FAKE, fv=FAKE)
    a.update(kw)
    return lib.lib.dsa_kpool_compress(a["k"], a["gate"], a["valid"], a["req_start"], a["B"], a["D"],
                                     a["kpool"], a["max_pools"], a["ape"], a["ln_w"], a["ln_b"],
                                     a["eps"], a["keys"], a["idx"], a["pv"], a["fv"], None)


def test_kpool_compress_refusals(B):
    assert _compress(B, kpool=9) == B.DSA_ERR_UNSUPPORTED        # KERNEL_MAX_KPOOL = 8
    assert _compress(B, kpool=0) == B.DSA_ERR_INVALID_ARG
    assert _compress(B, D=64) == B.DSA_ERR_UNSUPPORTED
    assert _compress(B, k=None) == B.DSA_ERR_INVALID_ARG
    assert _compress(B, k=FAKE + 8) == B.DSA_ERR_ALIGNMENT
    assert _compress(B, eps=-1.0) == B.DSA_ERR_INVALID_ARG
    assert _compress(B, eps=float("nan")) == B.DSA_ERR_INVALID_ARG
    assert _compress(B, B=0) == B.DSA_OK


def test_indexer_store_refusals(B):
    L = B.lib
    args = [FAKE, FAKE, None, FAKE, FAKE, 8, 128, FAKE, 2, FAKE, FAKE, FAKE, None]
    bad = list(args); bad[6] = 64
    assert L.dsa_indexer_store(*bad) == B.DSA_ERR_UNSUPPORTED        # D is the indexer dim 128
    bad = list(args); bad[5] = -1
    assert L.dsa_indexer_store(*bad) == B.DSA_ERR_INVALID_ARG
    bad = list(args); bad[0] = None
    assert L.dsa_indexer_store(*bad) == B.DSA_ERR_INVALID_ARG
    bad = list(args); bad[9] = None
    assert L.dsa_indexer_store(*bad) == B.DSA_ERR_INVALID_ARG       # no destination cache
    bad = list(args); bad[1] = FAKE + 4
    assert L.dsa_indexer_store(*bad) == B.DSA_ERR_ALIGNMENT
    bad = list(args); bad[3] = FAKE + 2
    assert L.dsa_indexer_store(*bad) == B.DSA_ERR_ALIGNMENT
    bad = list(args); bad[5] = 0
    assert L.dsa_indexer_store(*bad) == B.DSA_OK                     # nothing to store
    bad = list(args); bad[8] = 0; bad[7] = None; bad[9] = bad[10] = bad[11] = None
    assert L.dsa_indexer_store(*bad) == B.DSA_OK                     # no request to store into


def _compress_tokens(lib, **kw):
    a = dict(k=FAKE, gate=FAKE, valid=FAKE, req_start=FAKE, B=2, D=128, kpool=4, max_pools=8,
             ape=FAKE, ln_w=FAKE, ln_b=FAKE, eps=1e-5, tb=FAKE, te=FAKE, keys=FAKE, idx=FAKE,
             pv=FAKE, fv=FAKE)
    a.update(kw)
    return lib.lib.dsa_kpool_compress_tokens(
        a["k"], a["gate"], a["valid"], a["req_start"], a["B"], a["D"], a["kpool"], a["max_pools"],
        a["ape"], a["ln_w"], a["ln_b"], a["eps"], a["tb"], a["te"], a["keys"], a["idx"], a["pv"],
        a["fv"], None)


def test_kpool_compress_tokens_refusals(B):
    assert _compress_tokens(B, kpool=9) == B.DSA_ERR_UNSUPPORTED
    assert _compress_tokens(B, kpool=0) == B.DSA_ERR_INVALID_ARG
    assert _compress_tokens(B, D=256) == B.DSA_ERR_UNSUPPORTED
    assert _compress_tokens(B, tb=None) == B.DSA_ERR_INVALID_ARG
    assert _compress_tokens(B, te=None) == B.DSA_ERR_INVALID_ARG
    assert _compress_tokens(B, fv=None) == B.DSA_ERR_INVALID_ARG
    assert _compress_tokens(B, keys=None) == B.DSA_ERR_INVALID_ARG
    assert _compress_tokens(B, te=FAKE + 1) == B.DSA_ERR_ALIGNMENT
    assert _compress_tokens(B, eps=float("inf")) == B.DSA_ERR_INVALID_ARG
    assert _compress_tokens(B, max_pools=-1) == B.DSA_ERR_INVALID_ARG
    assert _compress_tokens(B, B=0) == B.DSA_OK


def test_index_scores_refusals(B):
    L = B.lib
    args = [FAKE, FAKE, FAKE, FAKE, 4, 16, 128, FAKE, FAKE, FAKE, 4, 4, 64, FAKE, FAKE, None]
    bad = list(args); bad[5] = 17
    assert L.dsa_index_scores(*bad) == B.DSA_ERR_UNSUPPORTED
    bad = list(args); bad[6] = 256
    assert L.dsa_index_scores(*bad) == B.DSA_ERR_UNSUPPORTED
    bad = list(args); bad[0] = None
    assert L.dsa_index_scores(*bad) == B.DSA_ERR_INVALID_ARG
    bad = list(args); bad[0] = FAKE + 2
    assert L.dsa_index_scores(*bad) == B.DSA_ERR_ALIGNMENT
    bad = list(args); bad[4] = 0
    assert L.dsa_index_scores(*bad) == B.DSA_OK


def test_topk_expand_refusals(B):
    L = B.lib
    args = [FAKE, FAKE, FAKE, FAKE, 4, 4, 64, 4, 16, FAKE, FAKE, None]
    bad = list(args); bad[8] = 4097
    assert L.dsa_topk_expand(*bad) == B.DSA_ERR_UNSUPPORTED
    bad = list(args); bad[7] = 9
    assert L.dsa_topk_expand(*bad) == B.DSA_ERR_UNSUPPORTED
    bad = list(args); bad[9] = None
    assert L.dsa_topk_expand(*bad) == B.DSA_ERR_INVALID_ARG
    bad = list(args); bad[8] = 0
    assert L.dsa_topk_expand(*bad) == B.DSA_OK


def test_topk_expand_tail_refusals(B):
    L = B.lib
    # scores, cand, pool_idx, q_req, q_pos, first_valid, tok_valid, req_start, Q, B, P, kpool, K
    args = [FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, 4, 64, 4, 16, FAKE, FAKE, None]
    bad = list(args); bad[11] = 0
    assert L.dsa_topk_expand_tail(*bad) == B.DSA_ERR_INVALID_ARG
    bad = list(args); bad[11] = 9
    assert L.dsa_topk_expand_tail(*bad) == B.DSA_ERR_UNSUPPORTED
    bad = list(args); bad[4] = None
    assert L.dsa_topk_expand_tail(*bad) == B.DSA_ERR_INVALID_ARG       # the tail needs q_pos
    bad = list(args); bad[5] = None
    assert L.dsa_topk_expand_tail(*bad) == B.DSA_ERR_INVALID_ARG       # ... and first_valid
    bad = list(args); bad[4] = FAKE + 2
    assert L.dsa_topk_expand_tail(*bad) == B.DSA_ERR_ALIGNMENT
    bad = list(args); bad[8] = 0
    assert L.dsa_topk_expand_tail(*bad) == B.DSA_OK
    # kpool 1 has no tail: select_k 0 then writes nothing at all
    bad = list(args); bad[11] = 1; bad[12] = 0
    assert L.dsa_topk_expand_tail(*bad) == B.DSA_OK


def test_sparse_mla_refusals(B):
    L = B.lib
    # partials of every split (the plan keeps the grid within 148 CTAs with at
    # least four 48-token chunks a split, half the row when it has fewer than
    # eight; 43 chunks for 2048 ids): 2 queries -> 11 splits of 4 chunks;
    # 16 queries -> 9 splits of 5 chunks; 1 query of 64 ids -> 2 splits of 1
    ws = B.dsa_sparse_mla_workspace_size(2, 64, 2048)
    assert ws == 2 * 11 * 64 * (512 * 2 + 8)
    assert B.dsa_sparse_mla_workspace_size(1, 16, 64) == 1 * 2 * 16 * (512 * 2 + 8)
    assert B.dsa_sparse_mla_workspace_size(16, 64, 2048) == 16 * 9 * 64 * (512 * 2 + 8)
    # at least 148 CTAs without splitting: one split, no workspace
    assert B.dsa_sparse_mla_workspace_size(148, 64, 2048) == 0
    assert B.dsa_sparse_mla_workspace_size(74, 128, 2048) == 0

    def call(**kw):
        a = dict(q=FAKE, kv=FAKE, rows=1 << 20, rs=FAKE, qr=FAKE, ids=FAKE, Q=2, B=2, Hm=64,
                 W=2048, lora=512, rope=0, scale=0.044, out=FAKE, lse=FAKE, ws=FAKE, wsb=ws)
        a.update(kw)
        return L.dsa_sparse_mla_decode(a["q"], a["kv"], a["rows"], a["rs"], a["qr"], a["ids"],
                                       a["Q"], a["B"], a["Hm"], a["W"], a["lora"], a["rope"],
                                       a["scale"], a["out"], a["lse"], a["ws"], a["wsb"], None)

    assert call(lora=576) == B.DSA_ERR_UNSUPPORTED      # KERNEL_KV_LORA_DIM = 512
    assert call(rope=64) == B.DSA_ERR_UNSUPPORTED       # NoPE only
    assert call(Hm=24) == B.DSA_ERR_UNSUPPORTED
    assert call(Hm=144) == B.DSA_ERR_UNSUPPORTED
    assert call(wsb=ws - 16) == B.DSA_ERR_WORKSPACE
    assert call(ws=None) == B.DSA_ERR_WORKSPACE
    assert call(q=None) == B.DSA_ERR_INVALID_ARG
    assert call(scale=float("inf")) == B.DSA_ERR_INVALID_ARG
    assert call(rows=-1) == B.DSA_ERR_INVALID_ARG
    assert call(rows=1 << 31) == B.DSA_ERR_UNSUPPORTED  # 32-bit row coordinates
    assert call(kv=None) == B.DSA_ERR_INVALID_ARG       # rows but no cache
    assert call(out=FAKE + 4) == B.DSA_ERR_ALIGNMENT
    assert call(Q=0) == B.DSA_OK


def test_paged_mla_refusals(B):
    L = B.lib
    # q, kv, kv_rows, table, max_blocks, page, seq_len, q_req, ids, Q, B, Hm, W, lora, rope, scale,
    # out, lse, ws, ws_bytes, stream
    args = [FAKE, FAKE, 1024, FAKE, 8, 16, FAKE, FAKE, FAKE, 2, 2, 64, 64, 512, 0, 0.04, FAKE,
            FAKE, FAKE, 1 << 30, None]
    bad = list(args); bad[5] = 0
    assert L.dsa_sparse_mla_decode_paged(*bad) == B.DSA_ERR_INVALID_ARG      # page size 0
    bad = list(args); bad[4] = -1
    assert L.dsa_sparse_mla_decode_paged(*bad) == B.DSA_ERR_INVALID_ARG
    bad = list(args); bad[6] = None
    assert L.dsa_sparse_mla_decode_paged(*bad) == B.DSA_ERR_INVALID_ARG      # no seq_len
    bad = list(args); bad[3] = FAKE + 2
    assert L.dsa_sparse_mla_decode_paged(*bad) == B.DSA_ERR_ALIGNMENT
    bad = list(args); bad[13] = 576
    assert L.dsa_sparse_mla_decode_paged(*bad) == B.DSA_ERR_UNSUPPORTED
    fp8 = args[:2] + [0.5] + args[2:]
    for s in (0.0, -1.0, float("inf"), float("nan")):
        bad = list(fp8); bad[2] = s
        assert L.dsa_sparse_mla_decode_paged_fp8(*bad) == B.DSA_ERR_INVALID_ARG
    bad = list(fp8); bad[10] = 0
    assert L.dsa_sparse_mla_decode_paged_fp8(*bad) == B.DSA_OK               # Q == 0


def test_indexer_select_refusals(B):
    L = B.lib
    #       hidden w     K     q_idx q_req q_pos Q  H   D    keys  pv    fv    pidx  B  kp mp    sk
    args = [FAKE, FAKE, 4096, FAKE, FAKE, FAKE, 4, 16, 128, FAKE, FAKE, FAKE, FAKE, 2, 4, 2048, 512,
            FAKE, FAKE, FAKE, FAKE, FAKE, None]
    bad = list(args); bad[7] = 17
    assert L.dsa_indexer_select(*bad) == B.DSA_ERR_UNSUPPORTED      # more than 16 heads
    bad = list(args); bad[8] = 64
    assert L.dsa_indexer_select(*bad) == B.DSA_ERR_UNSUPPORTED      # D is 128
    bad = list(args); bad[14] = 9
    assert L.dsa_indexer_select(*bad) == B.DSA_ERR_UNSUPPORTED      # kpool <= 8
    bad = list(args); bad[15] = 32769
    assert L.dsa_indexer_select(*bad) == B.DSA_ERR_UNSUPPORTED      # 8 CTAs x 4096 pools at most
    bad = list(args); bad[16] = 4097
    assert L.dsa_indexer_select(*bad) == B.DSA_ERR_UNSUPPORTED
    bad = list(args); bad[2] = 0
    assert L.dsa_indexer_select(*bad) == B.DSA_ERR_INVALID_ARG
    bad = list(args); bad[0] = None
    assert L.dsa_indexer_select(*bad) == B.DSA_ERR_INVALID_ARG
    bad = list(args); bad[21] = None
    assert L.dsa_indexer_select(*bad) == B.DSA_ERR_INVALID_ARG      # no token-id output
    bad = list(args); bad[3] = FAKE + 8
    assert L.dsa_indexer_select(*bad) == B.DSA_ERR_ALIGNMENT
    bad = list(args); bad[6] = 0
    assert L.dsa_indexer_select(*bad) == B.DSA_OK                   # Q == 0: nothing to do


def test_missing_library_fails_loudly(tmp_path, monkeypatch):
    """The binding has no fallback: without libdsa.so the import raises."""
    import importlib.util
    src = os.path.join(ROOT, "sparse_attention_indexer_head_b200", "binding.py")
    spec = importlib.util.spec_from_file_location("binding_copy", str(tmp_path / "binding.py"))
    (tmp_path / "binding.py").write_text(open(src).read())
    mod = importlib.util.module_from_spec(spec)
    with pytest.raises(ImportError):
        spec.loader.exec_module(mod)


def test_noalloc_scratch_covers_every_geometry(B):
    # The split geometry keeps every grid within one wave of 148 CTAs, so the
    # split-KV scratch of any call is at most 148 x 64 heads x (a bf16 row + m, l).
    bound = 148 * 64 * (512 * 2 + 8)
    assert bound <= B.DSA_NOALLOC_SCRATCH_BYTES
    # the binding reads the size from the library; it is the header's constant
    m = re.search(r"#define DSA_NOALLOC_SCRATCH_BYTES \((\d+)u << (\d+)\)", open(HEADER).read())
    assert m and B.DSA_NOALLOC_SCRATCH_BYTES == int(m.group(1)) << int(m.group(2))
    worst = 0
    for Q in list(range(1, 40)) + [64, 100, 147, 148, 149, 1000]:
        for hm in range(16, 129, 16):
            for W in (1, 31, 32, 33, 512, 2048, 4096 * 8, 1 << 20):
                n = B.dsa_sparse_mla_workspace_size(Q, hm, W)
                assert n % 16 == 0 and n <= bound, (Q, hm, W, n)
                worst = max(worst, n)
    assert worst > 0
