"""The in-tree builds decide staleness from a content hash of their inputs,
not from file times (a copied tree can round the times, which once made a
rebuilt source look older than a stale library).  No compiler runs here:
the hash and the up-to-date check are exercised on temporary files."""
import os
import threading
import time

from activation_residual_compression_cf_b200 import build as B


def test_stamp_tracks_content_not_file_times(tmp_path, monkeypatch):
    src = tmp_path / "k.cu"
    src.write_text("// v1\n")
    lib = tmp_path / "libx.so"
    lib.write_bytes(b"\x7fELF")
    monkeypatch.setattr(B, "LIB", str(lib))
    monkeypatch.setattr(B, "_deps", lambda: [str(src)])
    assert not B.up_to_date()                      # no stamp yet
    (tmp_path / "libx.so.sources").write_text(B._inputs_hash() + "\n")
    assert B.up_to_date()
    # a source edited with a time older than the library is still seen
    src.write_text("// v2\n")
    t = os.path.getmtime(lib) - 100
    os.utime(src, (t, t))
    assert not B.up_to_date()
    # and touching a file without changing it does not force a rebuild
    src.write_text("// v1\n")
    os.utime(src, None)
    assert B.up_to_date()


def test_hash_covers_flags_and_file_names(tmp_path, monkeypatch):
    a, b = tmp_path / "a.cu", tmp_path / "b.cu"
    a.write_text("x")
    b.write_text("x")
    monkeypatch.setattr(B, "_deps", lambda: [str(a)])
    h1 = B._inputs_hash()
    monkeypatch.setattr(B, "_deps", lambda: [str(b)])
    assert B._inputs_hash() != h1                  # same bytes, other file
    monkeypatch.setattr(B, "_deps", lambda: [str(a)])
    monkeypatch.setattr(B, "FLAGS", B.FLAGS + ["-DEXTRA"])
    assert B._inputs_hash() != h1                  # same file, other flags
    assert B._inputs_hash(debug=True) != B._inputs_hash()   # the debug build has its own stamp


def test_oracle_build_stamp(tmp_path, monkeypatch):
    from oracle import build as OB
    src = tmp_path / "o.c"
    src.write_text("int f(void){return 1;}\n")
    monkeypatch.setattr(OB, "SRC", str(src))
    h1 = OB._inputs_hash()
    src.write_text("int f(void){return 2;}\n")
    assert OB._inputs_hash() != h1


def test_concurrent_builds_take_turns(tmp_path, monkeypatch):
    """Ranks of a multi-GPU run that find the library stale at the same time
    compile one after another under the lock file, and the ones that get the
    lock after the first build find the library current and compile nothing
    (no two compilers write the same object files)."""
    monkeypatch.setattr(B, "ROOT", str(tmp_path))
    state = {"built": False, "active": 0, "most": 0, "compiles": 0}
    mu = threading.Lock()

    def fake_up_to_date(debug=False):
        return state["built"]

    def fake_compile(lib, verbose, debug):
        with mu:
            state["active"] += 1
            state["most"] = max(state["most"], state["active"])
        time.sleep(0.2)
        with mu:
            state["active"] -= 1
            state["compiles"] += 1
            state["built"] = True
        return lib

    monkeypatch.setattr(B, "up_to_date", fake_up_to_date)
    monkeypatch.setattr(B, "_compile", fake_compile)
    ts = [threading.Thread(target=B.build) for _ in range(4)]
    for t in ts:
        t.start()
    for t in ts:
        t.join()
    assert state["most"] == 1 and state["compiles"] == 1
