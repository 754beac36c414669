"""The C ABI without a GPU: the library loads, exports what include/h3attn.h
declares, and rejects bad arguments on the host before touching the device."""
import ctypes

import pytest

import video_diffusion_transformer_h3attn_b200 as h3
from video_diffusion_transformer_h3attn_b200 import _build

OK, INVALID, UNSUPPORTED, MISALIGNED = 0, 1, 2, 3
FAKE = 0x10000  # a 16-byte aligned address that is never dereferenced on the host


@pytest.fixture(scope="module")
def lib():
    _build.build()
    return h3.library()


def test_exports_every_declared_symbol(lib):
    names = h3.declared_symbols()
    assert set(names) >= {"h3attn_prologue", "h3attn_fwd", "h3attn_fwd_varlen", "h3attn_version",
                          "h3attn_status_string", "h3attn_last_error", "h3attn_device_status",
                          "h3attn_fwd_kv", "h3attn_merge", "h3attn_fwd_block_sparse", "h3attn_qkv_fused",
                          "h3attn_selftest_wait_timeout"}
    for n in names:
        assert hasattr(lib, n), "library does not export %s" % n


def test_version_and_status_strings(lib):
    assert lib.h3attn_version() >= 10000
    for code in range(6):
        assert lib.h3attn_status_string(code)
    assert lib.h3attn_status_string(99) == b"unknown status"


S3 = ctypes.c_int64 * 3
S2 = ctypes.c_int64 * 2


def fwd(lib, q=FAKE, k=FAKE, v=FAKE, o=FAKE, B=1, N=256, H=2, d=64, strides=(256 * 128, 128, 64),
        scale=0.0, lse=None):
    s = S3(*strides)
    return lib.h3attn_fwd(q, k, v, o, B, N, H, d, s, s, s, s, scale, lse, None)


def test_fwd_rejects_bad_arguments(lib):
    assert fwd(lib, q=None) == INVALID
    assert fwd(lib, d=96) == UNSUPPORTED
    assert fwd(lib, d=256) == UNSUPPORTED
    assert b"head_dim" in lib.h3attn_last_error()
    assert fwd(lib, H=0) == INVALID
    assert fwd(lib, N=0) == INVALID
    assert fwd(lib, B=0) == INVALID
    assert fwd(lib, q=FAKE + 2) == MISALIGNED
    assert fwd(lib, strides=(256 * 128, 130, 64)) == MISALIGNED
    assert fwd(lib, strides=(256 * 128, -128, 64)) == INVALID
    assert fwd(lib, scale=float("inf")) == INVALID
    assert fwd(lib, lse=FAKE + 2) == MISALIGNED
    assert b"lse" in lib.h3attn_last_error()


def varlen(lib, cu=FAKE, nseq=2, total=300, max_seqlen=200, H=2, d=128, strides=(256, 128)):
    s = S2(*strides)
    return lib.h3attn_fwd_varlen(FAKE, FAKE, FAKE, FAKE, cu, nseq, total, max_seqlen, H, d, s, s, s, s,
                                 0.0, None, None)


def test_varlen_rejects_bad_arguments(lib):
    assert varlen(lib, cu=None) == INVALID
    assert varlen(lib, nseq=0) == INVALID
    assert varlen(lib, total=0) == INVALID
    assert varlen(lib, max_seqlen=0) == INVALID
    assert varlen(lib, max_seqlen=301) == INVALID
    assert varlen(lib, d=80) == UNSUPPORTED
    assert varlen(lib, strides=(257, 128)) == MISALIGNED


def fwd_kv(lib, Nq=256, Nk=100, d=128, strides=(256 * 256, 256, 128), k=FAKE):
    s = S3(*strides)
    return lib.h3attn_fwd_kv(FAKE, k, FAKE, FAKE, 1, Nq, Nk, 2, d, s, s, s, s, 0.0, None, None)


def test_fwd_kv_rejects_bad_arguments(lib):
    assert fwd_kv(lib, Nq=0) == INVALID
    assert fwd_kv(lib, Nk=-1) == INVALID
    assert fwd_kv(lib, k=None) == INVALID
    assert fwd_kv(lib, k=FAKE + 2) == MISALIGNED
    assert fwd_kv(lib, d=32) == UNSUPPORTED
    assert fwd_kv(lib, Nk=(1 << 30) + 1) == UNSUPPORTED
    assert fwd_kv(lib, strides=(256 * 256, 252, 128)) == MISALIGNED


def fwd_sparse(lib, Nq=256, Nk=100, d=128, off=FAKE, idx=FAKE, k=FAKE):
    s = S3(256 * 256, 256, 128)
    return lib.h3attn_fwd_block_sparse(FAKE, k, FAKE, FAKE, 1, Nq, Nk, 2, d, s, s, s, s, off, idx, 0.0, None,
                                       None)


def test_fwd_block_sparse_rejects_bad_arguments(lib):
    assert fwd_sparse(lib, off=None) == INVALID
    assert fwd_sparse(lib, idx=None) == INVALID
    assert fwd_sparse(lib, off=FAKE + 2) == MISALIGNED
    assert fwd_sparse(lib, idx=FAKE + 6) == MISALIGNED
    assert fwd_sparse(lib, Nq=0) == INVALID
    assert fwd_sparse(lib, k=None) == INVALID
    assert fwd_sparse(lib, d=32) == UNSUPPORTED


def merge(lib, N=100, d=128, la=FAKE, o=FAKE, strides=(256 * 100, 256, 128), H=2):
    s = S3(*strides)
    return lib.h3attn_merge(FAKE, la, FAKE, FAKE, o, FAKE, 1, N, H, d, s, s, s, None)


def test_merge_rejects_bad_arguments(lib):
    assert merge(lib, la=None) == INVALID
    assert merge(lib, o=None) == INVALID
    assert merge(lib, N=-1) == INVALID
    assert merge(lib, H=0) == INVALID
    assert merge(lib, d=96) == UNSUPPORTED
    assert merge(lib, la=FAKE + 2) == MISALIGNED
    assert merge(lib, o=FAKE + 4) == MISALIGNED
    assert merge(lib, strides=(256 * 100, 260, 128)) == MISALIGNED
    assert merge(lib, N=0) == OK  # nothing to do: validated, nothing enqueued


def prologue(lib, n=10, H=2, d=128, gq=FAKE, pos=FAKE, kind=FAKE, sec=(32, 48, 48), eps=1e-6,
             theta=1e4, strides=(256, 128, 256, 128), q=FAKE):
    return lib.h3attn_prologue(q, FAKE, FAKE, FAKE, n, H, d, *strides, gq, FAKE, eps, pos, kind,
                               sec[0], sec[1], sec[2], theta, None)


def test_prologue_rejects_bad_arguments(lib):
    assert prologue(lib, q=None) == INVALID
    assert prologue(lib, d=96) == UNSUPPORTED
    assert prologue(lib, n=-1) == INVALID
    assert prologue(lib, H=0) == INVALID
    assert prologue(lib, sec=(32, 48, 50)) == INVALID      # does not sum to d
    assert prologue(lib, sec=(31, 49, 48)) == INVALID      # odd sections
    assert prologue(lib, kind=None) == INVALID              # pos without kind
    assert prologue(lib, theta=0.0) == INVALID
    assert prologue(lib, eps=-1.0) == INVALID
    assert prologue(lib, gq=FAKE + 8) == MISALIGNED
    assert prologue(lib, strides=(256, 128, 252, 128)) == MISALIGNED


def test_prologue_empty_is_a_no_op(lib):
    # zero tokens: validated, nothing enqueued, no device needed
    assert prologue(lib, n=0) == OK
    assert prologue(lib, n=0, pos=None, kind=None) == OK


def test_python_binding_refuses_cpu_tensors():
    torch = pytest.importorskip("torch")
    x = torch.zeros(4, 2, 64, dtype=torch.bfloat16)
    with pytest.raises(TypeError):
        h3.attention(x, x, x)
    with pytest.raises(TypeError):
        h3.prologue(x, x)


# ---- the Python binding's own checks, run on the host with stand-in CUDA tensors ----
# The binding must refuse an output that is too small (the kernels write every row
# through its strides) or on another device before anything reaches the library.
# Meta tensors wrapped to report a CUDA device stand in for device memory; the
# library is replaced by a stub that fails the test if a call gets through.

def _fake_cuda(torch, *shape, dtype=None, index=0):
    class _FakeCuda(torch.Tensor):
        @property
        def is_cuda(self):
            return True

        @property
        def device(self):
            return torch.device("cuda", index)

    return torch.Tensor._make_subclass(_FakeCuda, torch.empty(shape, dtype=dtype or torch.bfloat16, device="meta"))


@pytest.fixture
def no_library(monkeypatch):
    def refuse():
        raise AssertionError("the call reached the library")
    monkeypatch.setattr(h3, "library", refuse)


def test_binding_rejects_outputs_of_the_wrong_shape(no_library):
    torch = pytest.importorskip("torch")
    f = lambda *s, **kw: _fake_cuda(torch, *s, **kw)
    q = f(1, 300, 4, 128)
    for bad in (f(1, 200, 4, 128), f(1, 300, 2, 128), f(300, 4, 128), f(2, 300, 4, 128)):
        with pytest.raises(ValueError, match="o must have shape"):
            h3.attention(q, q, q, o=bad)
        with pytest.raises(ValueError, match="o must have shape"):
            h3.attention_kv(q, f(1, 50, 4, 128), f(1, 50, 4, 128), o=bad)
    with pytest.raises(ValueError, match="o must have shape"):
        h3.attention(q[0], q[0], q[0], o=f(299, 4, 128))
    qv = f(300, 4, 128)
    cu = f(3, dtype=torch.int32)
    with pytest.raises(ValueError, match="o must have shape"):
        h3.attention_varlen(qv, qv, qv, cu, 200, o=f(299, 4, 128))
    off = f(4 * 2 + 1, dtype=torch.int32)
    idx = f(10, dtype=torch.int32)
    with pytest.raises(ValueError, match="o must have shape"):
        h3.attention_block_sparse(q, q, q, off, idx, o=f(1, 256, 4, 128))
    lse = f(1, 4, 300, dtype=torch.float32)
    with pytest.raises(ValueError, match="o must have shape"):
        h3.merge(q, lse, q, lse, o=f(1, 300, 4, 64))
    x = f(300, 512)
    w = f(3 * 2 * 128, 512)
    with pytest.raises(ValueError, match="q_out must have shape"):
        h3.qkv_fused(x, w, 2, q_out=f(200, 2, 128))
    with pytest.raises(ValueError, match="k_out must have shape"):
        h3.prologue(qv, qv, f(300, 4, 128), f(300, 4, 64))


def test_binding_rejects_outputs_on_another_device(no_library):
    torch = pytest.importorskip("torch")
    q = _fake_cuda(torch, 1, 300, 4, 128)
    with pytest.raises(ValueError, match="cuda:1"):
        h3.attention(q, q, q, o=_fake_cuda(torch, 1, 300, 4, 128, index=1))
    with pytest.raises(ValueError, match="cuda:1"):
        h3.attention(q, _fake_cuda(torch, 1, 300, 4, 128, index=1), q)


def test_binding_checks_side_inputs_sizes(no_library):
    torch = pytest.importorskip("torch")
    f = lambda *s, **kw: _fake_cuda(torch, *s, **kw)
    qv, out = f(300, 4, 128), f(300, 4, 128)
    with pytest.raises(ValueError, match="gamma_q"):
        h3.prologue(qv, qv, out, out, gamma_q=f(64))
    with pytest.raises(ValueError, match="pos must be"):
        h3.prologue(qv, qv, out, out, pos=f(299, 3, dtype=torch.int32), kind=f(300, dtype=torch.uint8))
    with pytest.raises(ValueError, match="pos must be"):
        h3.prologue(qv, qv, out, out, pos=f(300, 3, dtype=torch.int32), kind=f(299, dtype=torch.uint8))
    x, w, o3 = f(300, 512), f(3 * 2 * 128, 512), f(300, 2, 128)
    with pytest.raises(ValueError, match="bias"):
        h3.qkv_fused(x, w, 2, bias=f(3 * 2 * 128 - 8), q_out=o3, k_out=o3, v_out=o3)


def test_binding_normalises_strides_of_size_one_dimensions():
    """A dimension of extent 1 is never stepped over, so a stride torch reports for
    it that the library would reject is passed as a valid one; the others as they are."""
    torch = pytest.importorskip("torch")
    from video_diffusion_transformer_h3attn_b200 import _strides2, _strides3
    t = torch.empty(1, 5, 4, 128).as_strided((1, 5, 4, 128), (0, 512, 128, 1))
    assert list(_strides3(t)) == [8, 512, 128]
    t = torch.empty(7, 1, 128).as_strided((7, 1, 128), (128, 3, 1))
    assert list(_strides2(t)) == [128, 8]
    t = torch.empty(2, 3, 4, 128)
    assert list(_strides3(t)) == [3 * 4 * 128, 4 * 128, 128]


def test_debug_bounds_build_exports_the_same_calls():
    """The bounds-checking debug build (H3ATTN_DEBUG_BOUNDS) exports every declared
    call and says so in its build flags; the release build does not."""
    import ctypes
    _build.build(debug_bounds=True)
    dbg = ctypes.CDLL(_build.DEBUG_LIBRARY)
    for n in h3.declared_symbols():
        assert hasattr(dbg, n), "debug library does not export %s" % n
    assert dbg.h3attn_build_flags() == 1
    assert h3.library().h3attn_build_flags() == 0
