"""CPU oracle for the SVG-EAR attention hot path (fp64, plain loops).

TEST INFRASTRUCTURE: only ``tests/``, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline / reference arm may import anything under this
package.  It shares no code with the CUDA path.
"""
