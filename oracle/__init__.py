"""CPU oracle for the rotated INT2 KV-cache hot path.

TEST INFRASTRUCTURE ONLY: imported by tests/, by __graft_entry__.smoke() and by
the CPU-baseline leg of bench.py, never by the product package.  The C file
kvq_oracle.c holds the arithmetic; oracle/oracle.py wraps it for numpy arrays;
oracle/np_mini.py is a second, independent numpy oracle used to cross-check
the first on tiny inputs.
"""
