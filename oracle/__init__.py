"""CSA2 CPU oracle — TEST INFRASTRUCTURE.

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg may import this
package. The product path (the CUDA library and its binding) never does.
"""
