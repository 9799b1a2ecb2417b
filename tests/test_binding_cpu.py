"""The Python binding's marshalling, checked on CPU against a stub library:
every wrapper passes the C function the arguments include/msa.h declares (in
number and order), byte counts for workspaces, and raises on a bad status."""
import ctypes

import pytest

import block_sparse_attention_decode_b200 as msa


class FakeTensor:
    """Stands in for a CUDA tensor: only what the binding reads."""

    def __init__(self, addr, numel=64, elsize=1):
        self.addr, self.n, self.es = addr, numel, elsize
        self.is_cuda = True
        self.dtype = None

    def data_ptr(self):
        return self.addr

    def numel(self):
        return self.n

    def element_size(self):
        return self.es


class FakeStream:
    cuda_stream = 0xABC0


class StubFn:
    def __init__(self, name, log, ret):
        self.name, self.log, self.ret = name, log, ret
        self.argtypes, self.restype = None, None

    def __call__(self, *args):
        self.log.append((self.name, args))
        return self.ret


class StubLib:
    def __init__(self, real, ret=0):
        self.log, self.real, self.ret = [], real, ret

    def __getattr__(self, name):
        if name == "msa_status_string":                      # host-only, safe to call
            return getattr(self.real, name)
        fn = StubFn(name, self.log, self.ret)
        fn.argtypes = getattr(self.real, name).argtypes       # the binding's declared types
        return fn


@pytest.fixture
def stub(monkeypatch):
    real = msa.load()
    lib = StubLib(real)
    monkeypatch.setattr(msa, "load", lambda: lib)
    return lib


def _objs():
    c = msa.msa_cache(idx_data=16, idx_scale=32, k_data=48, k_scale=64, v_data=80, v_scale=96,
                      s_idx=1.0, s_k=1.0, s_v=1.0, num_pages=4, idx_dtype=0)
    s = msa.msa_seqs(page_table=None, seq_lens=112, batch=1, q_tokens=1, max_pages=4)
    cache, seqs = msa.Cache.__new__(msa.Cache), msa.Seqs.__new__(msa.Seqs)
    cache.c, seqs.c = c, s
    return cache, seqs


def test_every_wrapper_matches_its_declaration(stub):
    cache, seqs = _objs()
    t = FakeTensor(0x1000)
    ws = FakeTensor(0x9000, numel=128, elsize=4)          # 512 bytes
    st = FakeStream()
    calls = [
        lambda: msa.msa_workspace_init(ws, st),
        lambda: msa.msa_indexer_score(cache, seqs, t, 1.0, None, t, ws, st),
        lambda: msa.msa_indexer_score_part(cache, seqs, t, 1.0, None, t, 1, 3, ws, st),
        lambda: msa.msa_block_maxpool_topk(t, True, seqs, t, ws, st),
        lambda: msa.msa_sparse_attn_decode(cache, seqs, t, 1.0, t, 0.1, t, ws, st),
        lambda: msa.msa_decode(cache, seqs, t, 1.0, t, 1.0, 0.1, t, None, ws, st),
        lambda: msa.msa_decode_static(cache, seqs, t, 1.0, t, 1.0, 0.1, t, None, st),
        lambda: msa.msa_debug_nvfp4_table(t, st),
    ]
    for call in calls:
        call()
    for name, args in stub.log:
        declared = getattr(stub.real, name).argtypes
        assert len(args) == len(declared), name
        if name != "msa_decode_static" and name != "msa_debug_nvfp4_table":
            ws_bytes = [a for a, ty in zip(args, declared) if ty is ctypes.c_size_t]
            assert ws_bytes == [512], (name, ws_bytes)
        assert args[-1].value == FakeStream.cuda_stream, name
    part_args = dict(stub.log)["msa_indexer_score_part"]
    assert (part_args[6], part_args[7]) == (1, 3)


def test_bad_status_raises(monkeypatch):
    real = msa.load()
    monkeypatch.setattr(msa, "load", lambda: StubLib(real, ret=msa.MSA_ERR_INVALID_ARG))
    cache, seqs = _objs()
    t = FakeTensor(0x1000)
    with pytest.raises(msa.MsaError) as e:
        msa.msa_decode(cache, seqs, t, 1.0, t, 1.0, 0.1, t, None, t, FakeStream())
    assert e.value.status == msa.MSA_ERR_INVALID_ARG


def test_kv_insert_rejects_non_bf16(stub):
    cache, seqs = _objs()
    t = FakeTensor(0x1000)
    with pytest.raises(ValueError):
        msa.msa_kv_insert(cache, seqs, t, t, t, t, FakeStream())


def test_declared_argument_counts_match_the_header():
    """The binding's ctypes argtypes have as many entries as the prototypes
    in include/msa.h have parameters."""
    import os
    import re
    hdr = open(os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                            "include", "msa.h")).read()
    hdr = re.sub(r"/\*.*?\*/", "", hdr, flags=re.S)
    protos = dict(re.findall(r"MSA_API\s+[\w\s\*]+?\b(msa_\w+)\s*\(([^)]*)\)\s*;", hdr))
    real = msa.load()
    assert set(msa.EXPORTED) <= set(protos)
    for name in msa.EXPORTED:
        params = protos[name].strip()
        n = 0 if params in ("", "void") else params.count(",") + 1
        assert len(getattr(real, name).argtypes) == n, name
