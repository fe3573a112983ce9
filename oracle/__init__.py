"""fp64 CPU oracle (test infrastructure only): ``ssm_oracle`` (numpy) and
``cref`` (plain C loaded with ctypes).  The product path never imports this."""
