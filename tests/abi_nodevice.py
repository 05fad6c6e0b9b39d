"""Calls into the C ABI from a child process that sees no CUDA device.

The host-side ABI tests pass made-up device addresses.  Arguments that pass
validation would reach a kernel launch if a device were current, so every
such call runs here, in a process started with CUDA_VISIBLE_DEVICES set to
the empty string: validation runs as usual, and a call that passes it stops
at the device check with MM_ERR_DEVICE.  Nothing is ever launched on a fake
address, on a GPU machine or off it.

The parent talks to one long-lived child over pipes: one JSON request per
line (entry point name and its arguments as integers or null) and one status
per line back.
"""

from __future__ import annotations

import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


class NoDeviceLib:
    """Proxy with the library's entry points as attributes; each call runs in
    the device-less child and returns its integer status."""

    def __init__(self):
        env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
        self._p = subprocess.Popen([sys.executable, os.path.abspath(__file__), "--serve"], cwd=ROOT, env=env,
                                   stdin=subprocess.PIPE, stdout=subprocess.PIPE, text=True, bufsize=1)
        ready = self._p.stdout.readline().strip()
        if ready != "ready":
            raise RuntimeError(f"ABI worker did not start: {ready!r}")

    def _call(self, name, args):
        self._p.stdin.write(json.dumps({"fn": name, "args": list(args)}) + "\n")
        self._p.stdin.flush()
        line = self._p.stdout.readline()
        if not line:
            raise RuntimeError("ABI worker exited")
        reply = json.loads(line)
        if "error" in reply:
            raise RuntimeError(reply["error"])
        return reply["status"]

    def setenv(self, name, value):
        """Set (or, with None, remove) an environment variable in the child."""
        self._p.stdin.write(json.dumps({"env": name, "value": value}) + "\n")
        self._p.stdin.flush()
        assert json.loads(self._p.stdout.readline()) == {"ok": True}

    def __getattr__(self, name):
        if not name.startswith("mamba_"):
            raise AttributeError(name)
        return lambda *args: self._call(name, args)

    def close(self):
        if self._p.poll() is None:
            self._p.stdin.close()
            self._p.wait(timeout=30)


def _serve():
    sys.path.insert(0, ROOT)
    assert os.environ.get("CUDA_VISIBLE_DEVICES") == "", "the worker must see no CUDA device"
    import mamba_selective_scan_core_b200 as mm

    L = mm.lib()
    print("ready", flush=True)
    for line in sys.stdin:
        req = json.loads(line)
        if "env" in req:
            if req["value"] is None:
                os.environ.pop(req["env"], None)
            else:
                os.environ[req["env"]] = str(req["value"])
            print(json.dumps({"ok": True}), flush=True)
            continue
        try:
            print(json.dumps({"status": int(getattr(L, req["fn"])(*req["args"]))}), flush=True)
        except Exception as e:  # reported to the parent, which raises
            print(json.dumps({"error": f"{type(e).__name__}: {e}"}), flush=True)


if __name__ == "__main__" and "--serve" in sys.argv:
    _serve()
